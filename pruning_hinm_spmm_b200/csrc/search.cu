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

#include <mutex>

#include "hinm_internal.h"
#include "launch.cuh"
#include "ptx.cuh"
#include "stage_rows.cuh"

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

// 2^e as an fp64, -1022 <= e <= 1023 (built from its bits; multiplying by it is exact).
__device__ __forceinline__ double pow2(int e) {
  return __longlong_as_double((long long)(1023 + e) << 52);
}

// Pass 1, thread per (tile, channel): V[t, c] = sum over the tile's rows, ascending, of
// I (fp64), and the tile's largest exponent P.
__global__ void vector_score_kernel(const ImpSrc src, int K, int T,
                                    double* __restrict__ Vc, int* __restrict__ tile_pmax) {
  ptx::enter_dependent();
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  int pm = 0;
  if (c < K) {
    const size_t row0 = (size_t)t * T;
    double acc = 0.0;
    uint32_t mb = 0;  // largest bit pattern = largest value (non-negative floats)
    constexpr int kBatch = 16;  // T is a multiple of 16
    float v[kBatch], nx[kBatch];
    const ImpColumn col = imp_column(src, K, c);
#pragma unroll
    for (int k = 0; k < kBatch; ++k) v[k] = col.at(row0 + k);
    for (int i0 = 0; i0 < T; i0 += kBatch) {
      // the next batch's loads go out before this batch's dependent chain
      if (i0 + kBatch < T) {
#pragma unroll
        for (int k = 0; k < kBatch; ++k) nx[k] = col.at(row0 + i0 + kBatch + k);
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {  // rows ascending
        acc = __dadd_rn(acc, (double)v[k]);
        mb = max(mb, __float_as_uint(v[k]));
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) v[k] = nx[k];
    }
    Vc[(size_t)t * K + c] = acc;
    if (mb) {
      uint32_t m;
      split_f32(__uint_as_float(mb), m, pm);
    }
  }
  for (int o = 16; o > 0; o >>= 1) pm = max(pm, __shfl_xor_sync(0xffffffffu, pm, o));
  if ((threadIdx.x & 31) == 0) atomicMax(tile_pmax + t, pm);
}

// Pass 2: each column's exact sum at the tile's scale, and a flag when some of its values
// fell below that scale (summed exactly elsewhere).  Two fp64 accumulators carry the common
// values exactly: level 1 takes p >= e1 = max(P - 22, lsb), level 2 takes p in [e2, e1) with
// e2 = max(e1 - 22, lsb).  At each level a value is an integer below 2^46 in units of
// 2^(level - 149), and a column has at most 128 values, so the fp64 sums stay integers below
// 2^53 and never round.  Smaller values (rare: 2^44 below the tile's largest) take a 128-bit
// integer path (p >= lsb) or set the flag.
//
// CTA of 256 threads per (tile, 256 channels): a thread takes 4 adjacent channels (one 16-byte
// load of I, or one 8-byte load of W, per row) over one of kSplit row ranges, with kBatch rows'
// loads in flight.  The rare path and the final combination of the row ranges go through
// shared memory (one 128-bit sum per (range, channel)), which keeps the registers to the fp64
// sums and the loads.
constexpr int kColThreads = 256;

// The rare values of a column (nonzero, below the second level) are only marked in the
// main pass; a second, out-of-line pass over the column's rows adds them exactly into its
// 128-bit sum in shared memory (p >= lsb, owner thread only) or sets the flag.  Both passes
// take the same values, so each value is counted once.
template <bool kW>
struct ImpQuad;
template <bool kW>
__device__ __noinline__ void col_rare_pass(const ImpQuad<kW> col, size_t row0, int rows, int j,
                                           float thr2, int lsb, U128* xs, unsigned char* tn) {
  U128 v = *xs;
  for (int i = 0; i < rows; ++i) {
    const float x = col.value(col.load(row0 + i), j);
    if (x >= thr2 || x == 0.0f) continue;
    uint32_t m;
    int e;
    split_f32(x, m, e);
    if (!m) continue;
    if (e >= lsb) add_shifted(v, m, e - lsb);
    else *tn = 1;
  }
  *xs = v;
}

// Channels c .. c + 3 (c a multiple of 4) of one row: the raw load (kW: 4 bf16 of W, else
// 4 fp32 of I), and value j of it as the importance.
template <>
struct ImpQuad<false> {
  using Raw = float4;
  const float* I;
  int K, c;
  __device__ __forceinline__ Raw load(size_t row) const {
    return __ldg(reinterpret_cast<const float4*>(I + row * K + c));
  }
  __device__ __forceinline__ float value(const Raw& r, int j) const {
    return j == 0 ? r.x : (j == 1 ? r.y : (j == 2 ? r.z : r.w));
  }
};
template <>
struct ImpQuad<true> {
  using Raw = uint2;
  const uint16_t* W;
  float s[4];
  int K, c;
  __device__ __forceinline__ Raw load(size_t row) const {
    return __ldg(reinterpret_cast<const uint2*>(W + row * K + c));
  }
  __device__ __forceinline__ float value(const Raw& r, int j) const {
    const uint32_t word = j < 2 ? r.x : r.y;
    return imp_from_w((j & 1) ? (word >> 16) : (word & 0xFFFFu), s[j]);
  }
};

// acc (units 2^(lsb - 149)) += a * 2^(e - lsb), a an fp64 integer below 2^53 in units
// 2^(e - 149), e - lsb <= 61
__device__ __forceinline__ void add_level(U128& acc, double a, int e, int lsb) {
  const unsigned long long ai = __double2ull_rz(__dmul_rn(a, pow2(149 - e)));
  const int sh = e - lsb;
  U128 f{ai << sh, sh ? (ai >> (64 - sh)) : 0ull};
  add128(acc, f);
}

template <int kBatch, int kSplit, bool kW>
__global__ void __launch_bounds__(kColThreads, 3) column_sum_kernel(
    const ImpSrc src, int K, int T, const int* __restrict__ tile_pmax,
    U128* __restrict__ colsum, unsigned char* __restrict__ coltiny) {
  ptx::enter_dependent();
  constexpr int kQuads = kColThreads / kSplit;  // channel quads per CTA
  __shared__ U128 xs[kSplit][kQuads * 4];
  __shared__ unsigned char tn[kSplit][kQuads * 4];
  const int q = threadIdx.x % kQuads, part = threadIdx.x / kQuads;
  const int c = (blockIdx.x * kQuads + q) * 4;
  const int t = blockIdx.y;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    xs[part][4 * q + k] = U128{0ull, 0ull};
    tn[part][4 * q + k] = 0;
  }
  const int pmax = tile_pmax[t];
  const int lsb = tile_lsb(pmax);
  const int e1 = max(pmax - 22, lsb), e2 = max(e1 - 22, lsb);
  const float thr1 = __uint_as_float((uint32_t)(e1 + 1) << 23);  // smallest fp32 with p >= e1
  const float thr2 = __uint_as_float((uint32_t)(e2 + 1) << 23);
  double a1[4] = {0.0, 0.0, 0.0, 0.0}, a2[4] = {0.0, 0.0, 0.0, 0.0};
  unsigned rare = 0u;  // bit j: channel c + j has values below the second level
  if (c < K) {  // K is a multiple of 4
    ImpQuad<kW> col;
    if constexpr (kW) {
      const float4 s4 = __ldg(reinterpret_cast<const float4*>(src.s + c));
      col = ImpQuad<kW>{src.W, {s4.x, s4.y, s4.z, s4.w}, K, c};
    } else {
      col = ImpQuad<kW>{src.I, K, c};
    }
    const int rows = T / kSplit;  // a multiple of kBatch
    const size_t row0 = (size_t)t * T + (size_t)part * rows;
    typename ImpQuad<kW>::Raw v[kBatch], nx[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) v[k] = col.load(row0 + k);
    for (int i0 = 0; i0 < rows; i0 += kBatch) {
      if (i0 + kBatch < rows) {  // next batch in flight during this one
#pragma unroll
        for (int k = 0; k < kBatch; ++k) nx[k] = col.load(row0 + i0 + kBatch + k);
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) {  // rows ascending
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float x = col.value(v[k], j);
          if (x >= thr1) {
            a1[j] = __dadd_rn(a1[j], (double)x);
          } else if (x >= thr2) {
            a2[j] = __dadd_rn(a2[j], (double)x);
          } else if (x != 0.0f) {
            rare |= 1u << j;
          }
        }
      }
#pragma unroll
      for (int k = 0; k < kBatch; ++k) v[k] = nx[k];
    }
    if (rare) {
      for (int j = 0; j < 4; ++j)
        if ((rare >> j) & 1u)
          col_rare_pass<kW>(col, row0, rows, j, thr2, lsb, &xs[part][4 * q + j], &tn[part][4 * q + j]);
    }
  }
  // this range's total per channel, then the ranges in order
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    U128 acc = xs[part][4 * q + j];
    add_level(acc, a1[j], e1, lsb);
    add_level(acc, a2[j], e2, lsb);
    xs[part][4 * q + j] = acc;
  }
  __syncthreads();
  if (part == 0 && c < K) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      U128 acc = xs[0][4 * q + j];
      unsigned char tiny = tn[0][4 * q + j];
#pragma unroll
      for (int r = 1; r < kSplit; ++r) {
        add128(acc, xs[r][4 * q + j]);
        tiny |= tn[r][4 * q + j];
      }
      colsum[(size_t)t * K + c + j] = acc;
      coltiny[(size_t)t * K + c + j] = tiny;
    }
  }
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

// Sorts one chunk of kRankChunk working positions of one tile by (key, index) ascending:
// a bitonic network with one element per thread; compare-exchange stages with partner
// distance < 32 run on warp shuffles, the wider ones through shared memory.
// zero64 / zero32 (nullptr allowed): buffers of a later kernel of the search, cleared here by
// the whole grid (grid-stride) instead of by separate memsets.
__global__ void __launch_bounds__(kRankChunk) chunk_sort_kernel(
    const double* __restrict__ Vc, const int32_t* __restrict__ perm, long long perm_stride,
    int K, int Kp,
    unsigned long long* __restrict__ skey, unsigned short* __restrict__ sidx,
    unsigned long long* __restrict__ zero64, size_t n64, int* __restrict__ zero32, size_t n32) {
  ptx::enter_dependent();
  __shared__ unsigned long long key_s[kRankChunk];
  __shared__ unsigned short idx_s[kRankChunk];
  {
    const size_t gt = ((size_t)blockIdx.y * gridDim.x + blockIdx.x) * kRankChunk + threadIdx.x;
    const size_t gs = (size_t)gridDim.x * gridDim.y * kRankChunk;
    if (zero64)
      for (size_t x = gt; x < n64; x += gs) zero64[x] = 0ull;
    if (zero32)
      for (size_t x = gt; x < n32; x += gs) zero32[x] = 0;
  }
  const int t = blockIdx.y, base = blockIdx.x * kRankChunk;
  const int i = threadIdx.x;
  const int j = base + i;
  unsigned long long key = ~0ull;
  unsigned idx = 0xFFFFu;
  if (j < K) {
    key = ~static_cast<unsigned long long>(
        __double_as_longlong(__ldg(Vc + (size_t)t * K +
                                   ptx::perm_at(perm ? perm + t * perm_stride : perm, j, K))));
    idx = (unsigned)j;
  }
  for (int k = 2; k <= kRankChunk; k <<= 1) {
    for (int jj = k >> 1; jj > 0; jj >>= 1) {
      const int l = i ^ jj;
      unsigned long long pk;
      unsigned pi;
      if (jj >= 32) {
        key_s[i] = key;
        idx_s[i] = (unsigned short)idx;
        __syncthreads();
        pk = key_s[l];
        pi = idx_s[l];
        __syncthreads();
      } else {
        pk = __shfl_xor_sync(0xffffffffu, key, jj);
        pi = __shfl_xor_sync(0xffffffffu, idx, jj);
      }
      const bool keep_min = ((i & k) == 0) == (i < l);
      const bool partner_less = pair_less(pk, pi, key, idx);
      if (partner_less == keep_min) {
        key = pk;
        idx = pi;
      }
    }
  }
  skey[(size_t)t * Kp + j] = key;
  sidx[(size_t)t * Kp + j] = (unsigned short)idx;
}

// rank[t][j] = number of (key, index) pairs of the tile below position j's.  One CTA per
// (tile, sorted chunk): all the tile's sorted chunks are copied into shared memory at once
// (every load in flight together); thread i takes the i-th pair of its own chunk (its rank
// within the chunk is i) and adds, for every other chunk, the number of that chunk's pairs
// below it (binary search; consecutive threads hold increasing pairs, so their searches
// follow nearly the same path).  The rank is then written at position j.
__global__ void __launch_bounds__(kRankChunk) merge_rank_kernel(
    const unsigned long long* __restrict__ skey, const unsigned short* __restrict__ sidx, int K,
    int Kp, int32_t* __restrict__ rank) {
  ptx::enter_dependent();
  extern __shared__ __align__(16) unsigned char merge_smem[];
  unsigned long long* ck = reinterpret_cast<unsigned long long*>(merge_smem);  // [Kp]
  unsigned short* ci = reinterpret_cast<unsigned short*>(ck + Kp);             // [Kp]
  const int t = blockIdx.y, own = blockIdx.x * kRankChunk;
  for (int q = threadIdx.x; q < Kp; q += kRankChunk) {
    ck[q] = __ldg(skey + (size_t)t * Kp + q);
    ci[q] = __ldg(sidx + (size_t)t * Kp + q);
  }
  __syncthreads();
  const unsigned long long kj = ck[own + threadIdx.x];
  const unsigned ij = ci[own + threadIdx.x];
  int r = threadIdx.x;
  for (int base = 0; base < Kp; base += kRankChunk) {
    if (base == own) continue;  // uniform over the CTA
    int lo = 0, hi = kRankChunk;  // count of pairs < (kj, ij) in this sorted chunk
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (pair_less(ck[base + mid], ci[base + mid], kj, ij)) lo = mid + 1;
      else hi = mid;
    }
    r += lo;
  }
  if (ij < (unsigned)K) rank[(size_t)t * K + ij] = r;  // padding pairs carry index 0xFFFF
}

size_t rank_scratch_bytes(int M, int K, int T) {
  const int nt = M / T;
  const size_t Kp = (size_t)((K + kRankChunk - 1) / kRankChunk) * kRankChunk;
  Carve c{nullptr, 0};
  c.take<unsigned long long>((size_t)nt * Kp);
  c.take<unsigned short>((size_t)nt * Kp);
  return (c.off + 255) & ~size_t(255);
}

namespace {

// V and the tile maxima (one launch after clearing the maxima).
cudaError_t launch_vector_scores(const ImpSrc& I, int M, int K, int T, double* V, int* tile_pmax,
                                 cudaStream_t s) {
  const int nt = M / T;
  cudaError_t e = cudaMemsetAsync(tile_pmax, 0, (size_t)nt * sizeof(int), s);
  if (e != cudaSuccess) return e;
  dim3 g1((K + 255) / 256, nt);
  return launch_kernel(vector_score_kernel, g1, 256, 0, s, nullptr, I, K, T, V, tile_pmax);
}

// The ranking from V: chunk sort, then merge.
cudaError_t launch_rank_sort(const double* V, const int32_t* perm, long long perm_stride, int M,
                             int K, int T,
                             int32_t* rank, void* scratch, cudaStream_t s,
                             unsigned long long* zero64 = nullptr, size_t n64 = 0,
                             int* zero32 = nullptr, size_t n32 = 0) {
  const int nt = M / T;
  cudaError_t e;
  const int nchunk = (K + kRankChunk - 1) / kRankChunk;
  const int Kp = nchunk * kRankChunk;
  Carve c{static_cast<char*>(scratch), 0};
  unsigned long long* skey = c.take<unsigned long long>((size_t)nt * Kp);
  unsigned short* sidx = c.take<unsigned short>((size_t)nt * Kp);
  e = launch_kernel(chunk_sort_kernel, dim3(nchunk, nt), kRankChunk, 0, s, nullptr, V, perm,
                    perm_stride, K, Kp, skey, sidx, zero64, n64, zero32, n32);
  if (e != cudaSuccess) return e;
  const size_t msmem = (size_t)Kp * (sizeof(unsigned long long) + sizeof(unsigned short));
  e = set_max_dynamic_smem((const void*)merge_rank_kernel, (int)msmem);
  if (e != cudaSuccess) return e;
  return launch_kernel(merge_rank_kernel, dim3(nchunk, nt), kRankChunk, msmem, s, nullptr, skey,
                       sidx, K, Kp, rank);
}

// A second stream per device for work that can run beside the caller's stream (forked and
// joined with events, so it also works under stream capture).  Created on the first call.
struct SideStream {
  cudaStream_t stream = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  void* ctx = nullptr;  // the context they were made in
};
constexpr int kMaxSideDevices = 64;
std::mutex g_side_mu;  // also orders the fork / join records of concurrent host threads
SideStream g_side[kMaxSideDevices];

cudaError_t side_stream(SideStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxSideDevices) return cudaErrorInvalidDevice;
  SideStream& ss = g_side[dev];
  void* ctx = current_cuda_context();
  // handles made in another context (the device's context was made again, e.g. after
  // cudaDeviceReset) went with it: make new ones in the current context
  if (ss.stream && ctx && ss.ctx && ctx != ss.ctx) ss = SideStream{};
  if (!ss.stream) {
    e = cudaStreamCreateWithFlags(&ss.stream, cudaStreamNonBlocking);
    if (e != cudaSuccess) return e;
    e = cudaEventCreateWithFlags(&ss.fork, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    e = cudaEventCreateWithFlags(&ss.join, cudaEventDisableTiming);
    if (e != cudaSuccess) return e;
    ss.ctx = ctx ? ctx : current_cuda_context();
  }
  *out = &ss;
  return cudaSuccess;
}

}  // namespace

cudaError_t launch_vector_rank(const ImpSrc& I, const int32_t* perm, long long perm_stride, int M,
                               int K, int T,
                               double* V, int32_t* rank, int* tile_pmax, void* scratch,
                               cudaStream_t s) {
  cudaError_t e = launch_vector_scores(I, M, K, T, V, tile_pmax, s);
  if (e != cudaSuccess) return e;
  return launch_rank_sort(V, perm, perm_stride, M, K, T, rank, scratch, s);
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

// value = v * 2^(lsb - 149) rounded to the nearest fp64, ties to even (the bucket-free case
// of exact_to_double, on two 64-bit words).
__device__ __forceinline__ double u128_to_double(U128 v, int lsb) {
  if (v.hi == 0ull && v.lo < (1ull << 53)) return ldexp((double)v.lo, lsb - 149);  // exact
  const int top = v.hi ? 127 - __clzll((long long)v.hi) : 63 - __clzll((long long)v.lo);
  const int lo = top - 52;  // keep bits [lo, lo + 53); lo >= 1 here
  unsigned long long mant;
  if (lo >= 64) mant = v.hi >> (lo - 64);
  else mant = (v.lo >> lo) | (v.hi << (64 - lo));
  mant &= (1ull << 53) - 1ull;
  const int hb = lo - 1;  // rounding bit
  const bool half = hb >= 64 ? ((v.hi >> (hb - 64)) & 1ull) : ((v.lo >> hb) & 1ull);
  bool sticky;  // any bit below hb
  if (hb >= 64) sticky = v.lo != 0ull || (hb > 64 && (v.hi & ((1ull << (hb - 64)) - 1ull)) != 0ull);
  else sticky = hb > 0 && (v.lo & ((1ull << hb) - 1ull)) != 0ull;
  int ex = lsb + lo - 149;
  if (half && (sticky || (mant & 1ull))) {
    mant += 1ull;
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
// position (block-wide prefix count), stored as their shared-memory slots stage_slot(c) in
// band_sum's staged rows -> band[t][m][q], and the exact sum of the dense
// vectors' column sums -> rdense[t][m] (values below the tile's scale go to the buckets).
template <int kPerMax>
__global__ void __launch_bounds__(512, 2) candidate_lists_kernel(
    const ImpSrc src, const int32_t* __restrict__ perm_all, long long perm_stride,
    const int32_t* __restrict__ rank,
    const int* __restrict__ tile_pmax, const U128* __restrict__ colsum,
    const unsigned char* __restrict__ coltiny, int K, int T, CandidateList cl, int ncand,
    unsigned short* __restrict__ band, U128* __restrict__ rdense,
    unsigned long long* __restrict__ bucket, int* __restrict__ bucket_used) {
  ptx::enter_dependent();
  __shared__ int warp_tot[16];
  __shared__ U128 warp_acc[16];
  const int m = blockIdx.x, t = blockIdx.y;
  const int32_t* perm = perm_all ? perm_all + t * perm_stride : perm_all;  // this tile's order
  const Candidate cand = cl.c[m];
  const int n4 = cand.n4, n24 = cand.n24;
  const int32_t* rk = rank + (size_t)t * K;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int lsb = tile_lsb(tile_pmax[t]);
  const size_t row0 = (size_t)t * T;
  unsigned long long* bkt = bucket + ((size_t)t * ncand + m) * 256;
  unsigned short* out = band + ((size_t)t * ncand + m) * K;
  U128 acc{0ull, 0ull};

  // each thread takes up to kPerMax consecutive working positions (kPerMax * 512 >= K);
  // the ranks stay in registers between the counting pass and the writing pass, and the
  // dependent loads of the second pass are issued kBatch positions at a time
  constexpr int kBatch = 4;
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * per, j1 = min(K, j0 + per);
  int rr[kPerMax];
#pragma unroll
  for (int q = 0; q < kPerMax; ++q) rr[q] = (q < per && j0 + q < j1) ? __ldg(rk + j0 + q) : -1;
  int cnt = 0;
#pragma unroll
  for (int q = 0; q < kPerMax; ++q) cnt += (rr[q] >= n4 && rr[q] < n4 + n24);
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
#pragma unroll
  for (int qb = 0; qb < kPerMax; qb += kBatch) {
    if (qb >= per) break;
    int c[kBatch];
    U128 cs[kBatch];
    unsigned char tn[kBatch];
#pragma unroll
    for (int q = 0; q < kBatch; ++q) c[q] = rr[qb + q] >= 0 ? ptx::perm_at(perm, j0 + qb + q, K) : 0;
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const bool dense = rr[qb + q] >= 0 && rr[qb + q] < n4;
      cs[q] = dense ? colsum[(size_t)t * K + c[q]] : U128{0ull, 0ull};
      tn[q] = dense ? coltiny[(size_t)t * K + c[q]] : (unsigned char)0;
    }
#pragma unroll
    for (int q = 0; q < kBatch; ++q) {
      const int r = rr[qb + q];
      if (r < 0) continue;
      if (r < n4) {
        add128(acc, cs[q]);
        if (tn[q]) {  // values below the tile's scale: exact buckets
          const ImpColumn col = imp_column(src, K, c[q]);
          for (int i = 0; i < T; ++i) {
            uint32_t mm;
            int e;
            split_f32(col.at(row0 + i), mm, e);
            if (mm && e < lsb) {
              atomicAdd(bkt + e, (unsigned long long)mm);
              used = true;
            }
          }
        }
      } else if (r < n4 + n24) {
        out[pos++] = (unsigned short)stage_slot(c[q]);
      }
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


// Loads RB consecutive floats (one channel's rows of the chunk) from shared memory.
template <int RB>
__device__ __forceinline__ void load_rows(const float* p, float (&v)[RB]) {
  if constexpr (RB == 8) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  } else if constexpr (RB == 4) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  } else if constexpr (RB == 2) {
    const float2 a = *reinterpret_cast<const float2*>(p);
    v[0] = a.x; v[1] = a.y;
  } else {
    v[0] = *p;
  }
}

// Exact sum of a value that missed the fast path (p < eb): to the tile-scale 128-bit sum
// `ex` when p >= lsb, else to the exponent buckets.
__device__ __forceinline__ void band_slow(float v, U128& ex, int lsb, unsigned long long* bkt,
                                          bool& used) {
  uint32_t m;
  int p;
  split_f32(v, m, p);
  if (!m) return;
  if (p >= lsb) {
    add_shifted(ex, m, p - lsb);
  } else {
    atomicAdd(bkt + p, (unsigned long long)m);
    used = true;
  }
}

// A group whose smaller top-2 value on some row lies below the fast path: each of its values
// to the fast sum or, below thr, to band_slow.  Out of line (rare), so that the common path
// stays short.
template <int RB>
struct GroupTop2 {
  float t1[RB], t2[RB];
};
struct BandSlowState {
  double acc;
  U128 ex;
  bool used;
};
template <int RB>
__device__ __noinline__ BandSlowState band_group_slow(const GroupTop2<RB> g, float thr,
                                                      BandSlowState st, int lsb,
                                                      unsigned long long* bkt) {
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    if (g.t1[r] >= thr) st.acc = __dadd_rn(st.acc, (double)g.t1[r]);
    else band_slow(g.t1[r], st.ex, lsb, bkt, st.used);
    if (g.t2[r] >= thr) st.acc = __dadd_rn(st.acc, (double)g.t2[r]);
    else band_slow(g.t2[r], st.ex, lsb, bkt, st.used);
  }
  return st;
}

// Per (tile, chunk of RB rows), 512 threads.  The chunk's rows of I are staged in shared
// memory channel-major (the RB values of channel c contiguous at slot stage_slot(c), one
// vector load each).  Then every candidate's 2:4 groups, as one candidate-major list, are
// split into equal contiguous slices, one per warp, and for every row the top 2 of each
// group's 4 values are summed.
//
// The sums are exact.  With eb = max(P - 24, lsb) every value with p >= eb is a multiple of
// u = 2^(eb - 149) below 2^48 u.  A lane adds at most 2 kG RB = 32 of them in fp64 per pass
// (kG groups), so that sum never rounds (an integer multiple of u below 2^53 u), in any
// order, and then moves it into a 64-bit integer.  Values with p < eb (rare: 2^24 below
// the tile's largest) go to band_slow.  Per (warp, candidate) the lanes' integers meet in
// three 21-bit-piece reductions and one shared atomic.
template <int RB, int kThreads>
__global__ void __launch_bounds__(kThreads) band_sum_kernel(
    const ImpSrc src, const unsigned short* __restrict__ band,
    const int* __restrict__ tile_pmax, int K, int T, CandidateList cl, int ncand,
    U128* __restrict__ part, unsigned long long* __restrict__ bucket,
    int* __restrict__ bucket_used) {
  ptx::enter_dependent();
  extern __shared__ __align__(16) float rows_s[];  // [K rounded up to 8][RB], stage_slot order
  __shared__ unsigned long long fast_sum[kMaxCandidates];   // units of 2^(eb - 149)
  __shared__ unsigned long long digits[kMaxCandidates][4];  // slow path, units of 2^(lsb - 149)
  const int chunk = blockIdx.x, t = blockIdx.y;
  const int nchunks = gridDim.x;
  const int lane = threadIdx.x & 31;
  const int K8 = (K + 7) & ~7;
  const int pmax = tile_pmax[t];
  const int lsb = tile_lsb(pmax);
  const int eb = max(pmax - 24, lsb);
  const float thr = __uint_as_float((uint32_t)(eb + 1) << 23);  // smallest fp32 with p >= eb
  const double unit_scale = pow2(149 - eb);                      // fp64 sum -> integer units
  for (int x = threadIdx.x; x < kMaxCandidates; x += kThreads) fast_sum[x] = 0ull;
  for (int x = threadIdx.x; x < kMaxCandidates * 4; x += kThreads) (&digits[0][0])[x] = 0ull;
  stage_rows_imp<RB, kThreads>(src, (size_t)t * T + (size_t)chunk * RB, K, rows_s);
  __syncthreads();

  const unsigned short* band_t = band + (size_t)t * ncand * K;
  // All candidates' groups form one list (candidate-major); warp w takes the contiguous
  // slice [w n / nwarps, (w + 1) n / nwarps) of it, so the warps' work is even and a warp
  // meets only the few candidates its slice spans.  Per candidate piece of the slice the
  // lanes take kG groups each per pass; after every pass a lane's fp64 sum (at most
  // 2 kG RB <= 32 values, exact) moves into its 64-bit integer sum, and at the end of the
  // piece the warp adds those with three 21-bit-piece reductions and one shared atomic.
  constexpr int kG = 4;
  constexpr int nwarps = kThreads / 32;
  const int warp = threadIdx.x >> 5;
  int total = 0;
  for (int m = 0; m < ncand; ++m) total += cl.c[m].n24 / 4;
  const int w0 = (int)((long long)total * warp / nwarps);
  const int w1 = (int)((long long)total * (warp + 1) / nwarps);
  int base = 0;  // first list index of candidate m
  for (int m = 0; m < ncand && base < w1; ++m) {
    const int ng = cl.c[m].n24 / 4;
    const int g0 = max(w0, base) - base, g1 = min(w1, base + ng) - base;
    base += ng;
    if (g0 >= g1) continue;  // warp-uniform: this candidate is outside the slice
    const ushort4* bl = reinterpret_cast<const ushort4*>(band_t + (size_t)m * K);
    unsigned long long* bkt = bucket + ((size_t)t * ncand + m) * 256;
    unsigned long long isum = 0ull;  // this lane's fast sum, integer units of 2^(eb - 149)
    U128 ex{0ull, 0ull};
    bool used = false;
    for (int gb = g0 + lane; gb < g1; gb += 32 * kG) {
      ushort4 cq[kG];
#pragma unroll
      for (int j = 0; j < kG; ++j)
        cq[j] = gb + 32 * j < g1 ? __ldg(bl + gb + 32 * j) : make_ushort4(0, 0, 0, 0);
      double acc = 0.0;
#pragma unroll
      for (int j = 0; j < kG; ++j) {
        if (gb + 32 * j >= g1) break;
        // the lists hold shared-memory slots (stage_slot of the channel), below K rounded up to 8
        float v0[RB], v1[RB], v2[RB], v3[RB];
        load_rows<RB>(rows_s + min((int)cq[j].x, K8 - 1) * RB, v0);
        load_rows<RB>(rows_s + min((int)cq[j].y, K8 - 1) * RB, v1);
        load_rows<RB>(rows_s + min((int)cq[j].z, K8 - 1) * RB, v2);
        load_rows<RB>(rows_s + min((int)cq[j].w, K8 - 1) * RB, v3);
        GroupTop2<RB> g2;
        float lo = INFINITY;
#pragma unroll
        for (int r = 0; r < RB; ++r) {
          const float a = fmaxf(v0[r], v1[r]), b = fminf(v0[r], v1[r]);
          const float cc = fmaxf(v2[r], v3[r]), d = fminf(v2[r], v3[r]);
          g2.t1[r] = fmaxf(a, cc);
          g2.t2[r] = fmaxf(fminf(a, cc), fmaxf(b, d));
          lo = fminf(lo, g2.t2[r]);
        }
        if (lo >= thr) {  // every value of the group on the fast path (t1 >= t2 >= thr)
          double g = 0.0;
#pragma unroll
          for (int r = 0; r < RB; ++r)
            g = __dadd_rn(g, __dadd_rn((double)g2.t1[r], (double)g2.t2[r]));
          acc = __dadd_rn(acc, g);
        } else {
          const BandSlowState st = band_group_slow<RB>(g2, thr, BandSlowState{acc, ex, used}, lsb, bkt);
          acc = st.acc;
          ex = st.ex;
          used = st.used;
        }
      }
      isum += __double2ull_rz(__dmul_rn(acc, unit_scale));  // an integer below 2^53
    }
    if (used) atomicOr(bucket_used + (size_t)t * ncand + m, 1);
    // the warp's fast sum (a lane's isum: at most 64 passes of < 2^53 each, < 2^59), in
    // three 21-bit pieces
    const unsigned s0 = __reduce_add_sync(0xffffffffu, (unsigned)(isum & 0x1FFFFFull));
    const unsigned s1 = __reduce_add_sync(0xffffffffu, (unsigned)((isum >> 21) & 0x1FFFFFull));
    const unsigned s2 = __reduce_add_sync(0xffffffffu, (unsigned)(isum >> 42));
    if (lane == 0) {
      const unsigned long long w = (unsigned long long)s0 + ((unsigned long long)s1 << 21) +
                                   ((unsigned long long)s2 << 42);
      if (w) atomicAdd(&fast_sum[m], w);
    }
    if (__any_sync(0xffffffffu, (ex.lo | ex.hi) != 0ull)) {
      for (int o = 16; o > 0; o >>= 1) {
        U128 other;
        other.lo = __shfl_xor_sync(0xffffffffu, ex.lo, o);
        other.hi = __shfl_xor_sync(0xffffffffu, ex.hi, o);
        add128(ex, other);
      }
      if (lane == 0) {
        atomicAdd(&digits[m][0], ex.lo & 0xFFFFFFFFull);
        atomicAdd(&digits[m][1], ex.lo >> 32);
        atomicAdd(&digits[m][2], ex.hi & 0xFFFFFFFFull);
        atomicAdd(&digits[m][3], ex.hi >> 32);
      }
    }
  }
  __syncthreads();
  if ((int)threadIdx.x < ncand) {
    // fold the digits' carries (each digit word is below 2^38: at most 32 warps add)
    const unsigned long long* d = digits[threadIdx.x];
    const unsigned long long d0 = d[0];
    const unsigned long long d1 = d[1] + (d0 >> 32);
    const unsigned long long d2 = d[2] + (d1 >> 32);
    const unsigned long long d3 = d[3] + (d2 >> 32);
    U128 tot;
    tot.lo = (d0 & 0xFFFFFFFFull) | (d1 << 32);
    tot.hi = (d2 & 0xFFFFFFFFull) | (d3 << 32);
    // + fast_sum * 2^(eb - lsb): fast_sum < 2^62 (a candidate has at most RB K / 2 <= 12288
    // values per CTA by band_config, each below 2^48 units), eb - lsb <= 59
    const unsigned long long f = fast_sum[threadIdx.x];
    const int sh = eb - lsb;
    U128 fx;
    fx.lo = f << sh;
    fx.hi = sh ? (f >> (64 - sh)) : 0ull;
    add128(tot, fx);
    part[((size_t)t * ncand + threadIdx.x) * nchunks + chunk] = tot;
  }
}

// Per tile, one warp per candidate: R(m) = exact total rounded once to fp64; then the
// first m with R(m+1) < R(m) (else the last candidate) gives the counts and v_s.
__global__ void finalize_kernel(const U128* __restrict__ rdense, const U128* __restrict__ part,
                                int nchunks, const unsigned long long* __restrict__ bucket,
                                const int* __restrict__ bucket_used,
                                const int* __restrict__ tile_pmax, int ncand, CandidateList cl,
                                double t_s, double alpha, double* __restrict__ R,
                                int32_t* __restrict__ counts, double* __restrict__ vs) {
  ptx::enter_dependent();
  __shared__ double Rs[kMaxCandidates];
  const int t = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  for (int m = warp; m < ncand; m += nwarps) {  // one warp per candidate
    const size_t tm = (size_t)t * ncand + m;
    U128 tot{0ull, 0ull};
    for (int c = lane; c < nchunks; c += 32) add128(tot, part[tm * nchunks + c]);
    for (int o = 16; o > 0; o >>= 1) {
      U128 other;
      other.lo = __shfl_xor_sync(0xffffffffu, tot.lo, o);
      other.hi = __shfl_xor_sync(0xffffffffu, tot.hi, o);
      add128(tot, other);
    }
    if (lane == 0) {
      add128(tot, rdense[tm]);
      const int lsb = tile_lsb(tile_pmax[t]);
      const double r = bucket_used[tm] ? exact_to_double(tot, lsb, bucket + tm * 256)
                                       : u128_to_double(tot, lsb);
      Rs[m] = r;
      R[tm] = r;
    }
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

// Rows and threads per band_sum CTA: the largest power of two <= 4 rows whose rows fit in
// 96 KB of shared memory, 512 threads, two CTAs per SM (T is a multiple of the rows; K <=
// 16384 keeps one row within 96 KB).  A thread then adds at most 32 values per candidate.
// (8 rows with 1024 threads, one CTA per SM, measured slower on the 4096-channel workload.)
struct BandCfg {
  int rows, threads;
};
static BandCfg band_config(int K) {
  const size_t K8 = ((size_t)K + 7) & ~size_t(7);  // stage_slot stays below K rounded up to 8
  int rb = 4;
  while (rb > 1 && (size_t)rb * K8 * sizeof(float) > 96u * 1024u) rb >>= 1;
  return {rb, 512};
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
  const int nchunks = T / band_config(K).rows;
  c.take<unsigned short>((size_t)nt * ncand * K);      // band channel lists
  c.take<U128>((size_t)nt * ncand);                    // dense exact sums
  c.take<U128>((size_t)nt * ncand * nchunks);          // 2:4 partial sums per row chunk
  c.take<unsigned long long>((size_t)nt * ncand * 256);  // exponent buckets
  c.take<int>((size_t)nt * ncand);                     // buckets used
  return (c.off + 255) & ~size_t(255);
}

cudaError_t launch_boundary_search(const ImpSrc& I, const void* stats, const int32_t* perm,
                                   long long perm_stride,
                                   int M, int K, int T, double t_s, double alpha,
                                   const Candidate* cands, int ncand, int32_t* counts_out,
                                   double* vs_out, int32_t* rank_out, double* retained_out,
                                   void* ws, int* status, cudaStream_t s) {
  (void)status;
  const int nt = M / T;
  Carve c{static_cast<char*>(ws), 0};
  double* V_ws = c.take<double>((size_t)nt * K);
  int32_t* rank_ws = c.take<int32_t>((size_t)nt * K);
  double* R_ws = c.take<double>((size_t)nt * ncand);
  double* R = retained_out ? retained_out : R_ws;
  int* pmax_ws = c.take<int>((size_t)nt);
  U128* colsum = c.take<U128>((size_t)nt * K);
  unsigned char* coltiny = c.take<unsigned char>((size_t)nt * K);
  char* rank_scratch = c.take<char>(rank_scratch_bytes(M, K, T));
  int32_t* rank = rank_out ? rank_out : rank_ws;
  // the candidates' buffers (same carving order as search_workspace_bytes)
  const BandCfg bc = band_config(K);
  const int RB = bc.rows;
  const int nchunks = T / RB;
  unsigned short* band = c.take<unsigned short>((size_t)nt * ncand * K);
  U128* rdense = c.take<U128>((size_t)nt * ncand);
  U128* part = c.take<U128>((size_t)nt * ncand * nchunks);
  unsigned long long* bucket = c.take<unsigned long long>((size_t)nt * ncand * 256);
  int* bucket_used = c.take<int>((size_t)nt * ncand);
  // V and the tile maxima: made with I by the importance step, or computed here
  const double* V = V_ws;
  const int* pmax = pmax_ws;
  cudaError_t e = cudaSuccess;
  if (stats) {
    V = static_cast<const double*>(stats);
    pmax = reinterpret_cast<const int*>(static_cast<const char*>(stats) +
                                        tile_stats_v_bytes(M, K, T));
  } else {
    e = launch_vector_scores(I, M, K, T, V_ws, pmax_ws, s);
    if (e != cudaSuccess) return e;
  }
  {
    // the exact column sums (which need the tile maxima) run on the side stream while the
    // ranking (which needs V) runs on the caller's stream; joined before the candidates
    std::lock_guard<std::mutex> lk(g_side_mu);
    SideStream* ss = nullptr;
    e = side_stream(&ss);
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(ss->fork, s);
    if (e != cudaSuccess) return e;
    e = cudaStreamWaitEvent(ss->stream, ss->fork, 0);
    if (e != cudaSuccess) return e;
    // a CTA per (tile, 256 channels); T = 64 splits its rows in 2, T = 128 in 4
    const dim3 gc((K + 255) / 256, nt);
    auto col = I.I ? (T == 128 ? column_sum_kernel<4, 4, false> : column_sum_kernel<4, 2, false>)
                   : (T == 128 ? column_sum_kernel<8, 4, true> : column_sum_kernel<8, 2, true>);
    // from I: 16-byte loads, 4 rows in flight; from W: 8-byte loads, 8 rows in flight
    e = launch_kernel(col, gc, kColThreads, 0, ss->stream, nullptr, I, K, T, pmax, colsum,
                      coltiny);
    if (e != cudaSuccess) return e;
    e = cudaEventRecord(ss->join, ss->stream);
    if (e != cudaSuccess) return e;
    // the sort also clears the exponent buckets and their flags (used from candidate_lists on)
    e = launch_rank_sort(V, perm, perm_stride, M, K, T, rank, rank_scratch, s, bucket,
                         (size_t)nt * ncand * 256, bucket_used, (size_t)nt * ncand);
    if (e != cudaSuccess) return e;
    e = cudaStreamWaitEvent(s, ss->join, 0);
    if (e != cudaSuccess) return e;
  }
  CandidateList cl;
  for (int i = 0; i < kMaxCandidates; ++i) cl.c[i] = i < ncand ? cands[i] : Candidate{0, 0, 0};
  {
    const dim3 gl(ncand, nt);
    const int per = (K + 511) / 512;
    auto lists = per <= 8 ? candidate_lists_kernel<8>
                          : (per <= 16 ? candidate_lists_kernel<16> : candidate_lists_kernel<32>);
    e = launch_kernel(lists, gl, 512, 0, s, nullptr, I, perm, perm_stride, rank, pmax, colsum,
                      coltiny, K, T, cl, ncand, band, rdense, bucket, bucket_used);
  }
  if (e != cudaSuccess) return e;
  const size_t smem = (size_t)RB * (((size_t)K + 7) & ~size_t(7)) * sizeof(float);
  for (const void* fn : {(const void*)band_sum_kernel<1, 512>, (const void*)band_sum_kernel<2, 512>,
                         (const void*)band_sum_kernel<4, 512>}) {
    e = set_max_dynamic_smem(fn, 96 * 1024);
    if (e != cudaSuccess) return e;
  }
  const dim3 gb(nchunks, nt);
  auto sum = RB == 4 ? band_sum_kernel<4, 512>
                     : (RB == 2 ? band_sum_kernel<2, 512> : band_sum_kernel<1, 512>);
  e = launch_kernel(sum, gb, 512, smem, s, nullptr, I, band, pmax, K, T, cl, ncand, part, bucket,
                    bucket_used);
  if (e != cudaSuccess) return e;
  return launch_kernel(finalize_kernel, nt, 1024, 0, s, nullptr, rdense, part, nchunks, bucket,
                       bucket_used, pmax, ncand, cl, t_s, alpha, R, counts_out, vs_out);
}

}  // namespace hinm
