// a4. Mask: regions by rank, 2:4 groups in ascending working position, top-2 of 4 per
// row (FlexHiNM-GP notes, 亮点与洞察: high -> dense, middle -> 2:4, low -> pruned;
// rkmt.cn section 二: keep 2 of every 4 consecutive; geek-doc.cn section 五: the mask has
// W's shape).
//
//   classify_kernel       one CTA per tile: region of every working position and the
//                         2:4 members' input channels in ascending working position
//                         (member[t][q])
//   bitmask_kernel        one CTA per (tile, RB <= 8 rows): the rows staged channel-major
//                         in shared memory (16-byte quad loads), keep bytes (dense channels
//                         all rows, 2:4 groups top-2 of 4 per row), then the bitmask words
//                         assembled by warp ballots and written once, coalesced.
#include <cuda_runtime.h>

#include "hinm_internal.h"
#include "launch.cuh"
#include "ptx.cuh"
#include "stage_rows.cuh"

namespace hinm {

// Block-wide exclusive scan of one int per thread (blockDim.x <= 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_tot, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int x = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += x;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int nw = (blockDim.x + 31) >> 5;
    int w = lane < nw ? warp_tot[lane] : 0;
    int wi = w;
    for (int o = 1; o < 32; o <<= 1) {
      const int x = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += x;
    }
    if (lane < nw) warp_tot[lane] = wi - w;
    if (lane == 31) *total = wi;
  }
  __syncthreads();
  const int r = warp_tot[warp] + incl - v;
  __syncthreads();
  return r;
}

__global__ void __launch_bounds__(1024) classify_kernel(const int32_t* __restrict__ rank,
                                                        const int32_t* __restrict__ perm_all,
                                                        long long perm_stride,
                                                        const int32_t* __restrict__ counts, int K,
                                                        int8_t* __restrict__ region,
                                                        int32_t* __restrict__ member,
                                                        int* status) {
  ptx::enter_dependent();
  __shared__ int warp_tot[32];
  __shared__ int total;
  __shared__ uint32_t seen[kMaxK / 32];  // which channels this tile's order has named
  const int t = blockIdx.x;
  const int32_t* perm = perm_all ? perm_all + t * perm_stride : perm_all;  // this tile's order
  if ((t == 0 || perm_stride != 0) && perm) {
    // the permutation must name every channel 0..K-1 once: a repeated or out-of-range
    // entry is reported as HINM_ERR_INVALID_ARG (perm_at keeps every access in range)
    for (int w = threadIdx.x; w < kMaxK / 32; w += blockDim.x) seen[w] = 0u;
    __syncthreads();
    for (int j = threadIdx.x; j < K; j += blockDim.x) {
      const int c = __ldg(perm + j);
      if (c < 0 || c >= K) {
        ptx::record_status(status, HINM_ERR_INVALID_ARG);
      } else {
        const uint32_t bit = 1u << (c & 31);
        if (atomicOr(seen + (c >> 5), bit) & bit) ptx::record_status(status, HINM_ERR_INVALID_ARG);
      }
    }
  }
  int n0 = counts[3 * t], n24 = counts[3 * t + 1], n4 = counts[3 * t + 2];
  if (n0 < 0 || n24 < 0 || n4 < 0 || n0 + n24 + n4 != K || (n24 & 3)) {
    if (threadIdx.x == 0) ptx::record_status(status, HINM_ERR_INVALID_ARG);
    n24 = 0;
    n4 = 0;
  }
  const int32_t* rk = rank + (size_t)t * K;
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * per, j1 = min(K, j0 + per);
  int cnt = 0;
  for (int j = j0; j < j1; ++j) {
    const int r = rk[j];
    cnt += (r >= n4 && r < n4 + n24);
  }
  int pos = block_exclusive_scan(cnt, warp_tot, &total);
  int8_t* reg = region + (size_t)t * K;
  int32_t* mem = member + (size_t)t * K;
  for (int j = j0; j < j1; ++j) {
    const int r = rk[j];
    const int c = ptx::perm_at(perm, j, K);
    int8_t cls = HINM_REGION_PRUNED;
    if (r < n4) {
      cls = HINM_REGION_DENSE;
    } else if (r < n4 + n24) {
      cls = HINM_REGION_24;
      mem[pos++] = c;
    }
    reg[c] = cls;
  }
}

// One CTA per (tile, RB rows).  The rows of I are staged channel-major in shared memory
// (the RB values of channel c contiguous).  keep[c] holds one bit per row: all ones for a
// dense channel, zero for a pruned one, and for a 2:4 channel the rows where it is among
// the top 2 of its group (ties: the lower working position wins).  Each channel belongs
// to one group, so every keep byte has one writer.  The mask words are then assembled by
// warp ballots, 32 words per warp and row, and stored coalesced.
constexpr int kMaskThreads = 512;

template <int RB>
__device__ __forceinline__ void mask_load_rows(const float* p, float (&v)[RB]) {
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

// Keep bits of a 2:4 group's four members over RB rows (v[k][r]: member k's value in row r).
// g_kl bit r: member l beats member k (k < l) in row r, i.e. v_l > v_k (equal values: the
// lower position k wins).  Member k is kept iff at most one member beats it: the negated
// majority of its three "beaten by" words, all rows at once.
template <int RB>
__device__ __forceinline__ void group_keep(const float (&v)[4][RB], uint32_t (&kb)[4]) {
  uint32_t g01 = 0u, g02 = 0u, g03 = 0u, g12 = 0u, g13 = 0u, g23 = 0u;
#pragma unroll
  for (int r = 0; r < RB; ++r) {
    g01 |= (uint32_t)(v[1][r] > v[0][r]) << r;
    g02 |= (uint32_t)(v[2][r] > v[0][r]) << r;
    g03 |= (uint32_t)(v[3][r] > v[0][r]) << r;
    g12 |= (uint32_t)(v[2][r] > v[1][r]) << r;
    g13 |= (uint32_t)(v[3][r] > v[1][r]) << r;
    g23 |= (uint32_t)(v[3][r] > v[2][r]) << r;
  }
  auto maj = [](uint32_t a, uint32_t b, uint32_t c) { return (a & b) | (a & c) | (b & c); };
  constexpr uint32_t kRows = (1u << RB) - 1u;
  kb[0] = ~maj(g01, g02, g03) & kRows;
  kb[1] = ~maj(~g01, g12, g13) & kRows;
  kb[2] = ~maj(~g02, ~g12, g23) & kRows;
  kb[3] = ~maj(~g03, ~g13, ~g23) & kRows;
}

// Dense channels keep every row: keep[c] = all ones for them, 0 for the others (4 channels
// per thread, K % 4 == 0).
template <int RB>
__device__ __forceinline__ void keep_dense(const int8_t* __restrict__ reg, int K, uint8_t* keep) {
  constexpr uint8_t kAll = (uint8_t)((1u << RB) - 1u);
  for (int q = threadIdx.x; q < (K >> 2); q += kMaskThreads) {
    const char4 rq = __ldg(reinterpret_cast<const char4*>(reg) + q);
    const uint32_t k4 = (rq.x == HINM_REGION_DENSE ? (uint32_t)kAll : 0u) |
                        (rq.y == HINM_REGION_DENSE ? (uint32_t)kAll << 8 : 0u) |
                        (rq.z == HINM_REGION_DENSE ? (uint32_t)kAll << 16 : 0u) |
                        (rq.w == HINM_REGION_DENSE ? (uint32_t)kAll << 24 : 0u);
    reinterpret_cast<uint32_t*>(keep)[q] = k4;
  }
}

// The tile's 2:4 group count from the counts (0 when they are not a valid split of K).
__device__ __forceinline__ int groups_24(const int32_t* counts, int t, int K) {
  int n24 = counts[3 * t + 1];
  const int n0 = counts[3 * t], n4 = counts[3 * t + 2];
  if (n0 < 0 || n24 < 0 || n4 < 0 || n0 + n24 + n4 != K || (n24 & 3)) n24 = 0;
  return n24 / 4;
}

// The mask words of RB rows from their keep bytes (bit r of keep[c] = row r keeps channel
// c): 32 words per warp and row by ballots, stored coalesced.
template <int RB>
__device__ __forceinline__ void write_words(const uint8_t* keep, int K, uint32_t* out) {
  const int words = (K + 31) >> 5;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int nwarps = kMaskThreads / 32;
  for (int wb = warp * 32; wb < words; wb += nwarps * 32) {
    uint32_t mine[RB];
#pragma unroll
    for (int r = 0; r < RB; ++r) mine[r] = 0u;
    const int nw = min(32, words - wb);
    for (int i = 0; i < nw; ++i) {
      const int c = (wb + i) * 32 + lane;
      const uint32_t kbyte = c < K ? keep[c] : 0u;
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        const uint32_t bits = __ballot_sync(0xffffffffu, (kbyte >> r) & 1u);
        if (lane == i) mine[r] = bits;
      }
    }
    if (lane < nw) {
#pragma unroll
      for (int r = 0; r < RB; ++r) out[(size_t)r * words + wb + lane] = mine[r];
    }
  }
}

template <int RB>
__global__ void __launch_bounds__(kMaskThreads) bitmask_kernel(
    const ImpSrc src, const int8_t* __restrict__ region, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ member, int K, int T, uint32_t* __restrict__ bitmask) {
  ptx::enter_dependent();
  extern __shared__ __align__(16) uint8_t mask_smem[];
  const int K8 = (K + 7) & ~7;
  float* rows_s = reinterpret_cast<float*>(mask_smem);  // [K8][RB], stage_slot order
  uint8_t* keep = mask_smem + (size_t)K8 * RB * sizeof(float);
  const int words = (K + 31) >> 5;
  const int t = blockIdx.y;
  const int r0 = blockIdx.x * RB;  // first row of the chunk within the tile
  const int8_t* reg = region + (size_t)t * K;
  stage_rows_imp<RB, kMaskThreads>(src, (size_t)t * T + r0, K, rows_s);
  keep_dense<RB>(reg, K, keep);
  __syncthreads();

  const int ng = groups_24(counts, t, K);
  const int32_t* mem = member + (size_t)t * K;
  for (int g = threadIdx.x; g < ng; g += kMaskThreads) {
    // the group's input channels, in ascending working position (k = 0..3)
    const int4 cq = __ldg(reinterpret_cast<const int4*>(mem) + g);
    const int cc[4] = {cq.x, cq.y, cq.z, cq.w};
    int c[4];
    float v[4][RB];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      c[k] = ((unsigned)cc[k] < (unsigned)K) ? cc[k] : 0;  // never index outside I
      mask_load_rows<RB>(rows_s + (size_t)stage_slot(c[k]) * RB, v[k]);
    }
    uint32_t kb[4];
    group_keep<RB>(v, kb);
#pragma unroll
    for (int k = 0; k < 4; ++k) keep[c[k]] = (uint8_t)kb[k];
  }
  __syncthreads();
  write_words<RB>(keep, K, bitmask + ((size_t)t * T + r0) * words);
}

// The same mask from W without a materialized I: the chunk's RB rows of W (bf16) are copied
// into shared memory as they are (cp.async, no conversion), and only the 2:4 groups'
// members are turned into importances, fl32(fl32(w^2) s_c) as the importance kernels round
// them, where they are compared; dense and pruned channels need no value.
template <int RB>
__global__ void __launch_bounds__(kMaskThreads) bitmask_w_kernel(
    const uint16_t* __restrict__ W, const float* __restrict__ s_c,
    const int8_t* __restrict__ region, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ member, int K, int T, uint32_t* __restrict__ bitmask) {
  ptx::enter_dependent();
  extern __shared__ __align__(16) uint8_t mask_smem[];
  const int K8 = (K + 7) & ~7;  // row stride in shared memory (16-byte rows)
  uint16_t* w_s = reinterpret_cast<uint16_t*>(mask_smem);  // [RB][K8]
  uint8_t* keep = mask_smem + (size_t)RB * K8 * sizeof(uint16_t);
  const int words = (K + 31) >> 5;
  const int t = blockIdx.y;
  const int r0 = blockIdx.x * RB;
  const int8_t* reg = region + (size_t)t * K;
  {
    const uint32_t dst = ptx::smem_u32(w_s);
    for (int a = 0; a < RB; ++a) {
      const uint16_t* src = W + ((size_t)t * T + r0 + a) * K;
      const uint32_t rd = dst + (uint32_t)(a * K8 * 2);
      if ((K & 7) == 0) {
        for (int q = threadIdx.x; q < (K >> 3); q += kMaskThreads) ptx::cp_async16(rd + 16 * q, src + 8 * q);
      } else {
        for (int q = threadIdx.x; q < (K >> 2); q += kMaskThreads) ptx::cp_async8(rd + 8 * q, src + 4 * q);
      }
    }
  }
  keep_dense<RB>(reg, K, keep);  // while the rows land
  ptx::cp_async_commit_wait_all();
  __syncthreads();

  const int ng = groups_24(counts, t, K);
  const int32_t* mem = member + (size_t)t * K;
  for (int g = threadIdx.x; g < ng; g += kMaskThreads) {
    const int4 cq = __ldg(reinterpret_cast<const int4*>(mem) + g);
    const int cc[4] = {cq.x, cq.y, cq.z, cq.w};
    int c[4];
    float sk[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      c[k] = ((unsigned)cc[k] < (unsigned)K) ? cc[k] : 0;  // never index outside W
      sk[k] = __ldg(s_c + c[k]);
    }
    float v[4][RB];
#pragma unroll
    for (int k = 0; k < 4; ++k)
#pragma unroll
      for (int r = 0; r < RB; ++r) v[k][r] = imp_from_w(w_s[r * K8 + c[k]], sk[k]);
    uint32_t kb[4];
    group_keep<RB>(v, kb);
#pragma unroll
    for (int k = 0; k < 4; ++k) keep[c[k]] = (uint8_t)kb[k];
  }
  __syncthreads();
  write_words<RB>(keep, K, bitmask + ((size_t)t * T + r0) * words);
}

// Rows per bitmask CTA: the largest power of two <= 8 whose rows fit in 96 KB of shared
// memory (T is a multiple of it), so that wide rows (K ~ 11008) still get two per CTA.
static int mask_rows(int K) {
  const size_t K8 = ((size_t)K + 7) & ~size_t(7);
  int rb = 8;
  while (rb > 1 && (size_t)rb * K8 * sizeof(float) > 96u * 1024u) rb >>= 1;
  return rb;
}

// Rows per CTA of the W-path mask: the largest of 8, 4, 2 whose bf16 rows fit in 96 KB of
// shared memory (K <= 16384 always fits 2).
static int mask_rows_w(int K) {
  const size_t K8 = ((size_t)K + 7) & ~size_t(7);
  int rb = 8;
  while (rb > 2 && (size_t)rb * K8 * sizeof(uint16_t) > 96u * 1024u) rb >>= 1;
  return rb;
}

size_t mask_workspace_bytes(int M, int K, int T) {
  const int nt = M / T;
  Carve c{nullptr, 0};
  c.take<double>((size_t)nt * K);   // V (only when no rank is passed)
  c.take<int32_t>((size_t)nt * K);  // rank (only when no rank is passed)
  c.take<int32_t>((size_t)nt * K);  // member
  c.take<int>((size_t)nt);          // tile max exponent (by-product of the ranking)
  c.take<char>(rank_scratch_bytes(M, K, T));
  return (c.off + 255) & ~size_t(255);
}

cudaError_t launch_mask(const ImpSrc& I, const int32_t* perm, long long perm_stride,
                        const int32_t* counts,
                        const int32_t* rank, int M, int K, int T, uint32_t* bitmask,
                        int8_t* region, void* ws, int* status, cudaStream_t s) {
  const int nt = M / T;
  Carve cv{static_cast<char*>(ws), 0};
  double* V = cv.take<double>((size_t)nt * K);
  int32_t* rank_ws = cv.take<int32_t>((size_t)nt * K);
  int32_t* member = cv.take<int32_t>((size_t)nt * K);
  int* pmax = cv.take<int>((size_t)nt);
  char* rank_scratch = cv.take<char>(rank_scratch_bytes(M, K, T));
  cudaError_t e;
  if (!rank) {
    e = launch_vector_rank(I, perm, perm_stride, M, K, T, V, rank_ws, pmax, rank_scratch, s);
    if (e != cudaSuccess) return e;
    rank = rank_ws;
  }
  e = launch_kernel(classify_kernel, nt, 1024, 0, s, nullptr, rank, perm, perm_stride, counts, K,
                    region, member, status);
  if (e != cudaSuccess) return e;
  if (!I.I) {  // from W: rows copied as bf16, importances only for the compared members
    const int RB = mask_rows_w(K);
    const size_t smem = (size_t)RB * (((size_t)K + 7) & ~size_t(7)) * sizeof(uint16_t) + (size_t)K;
    for (const void* fn : {(const void*)bitmask_w_kernel<2>, (const void*)bitmask_w_kernel<4>,
                           (const void*)bitmask_w_kernel<8>}) {
      e = set_max_dynamic_smem(fn, 96 * 1024 + kMaxK);
      if (e != cudaSuccess) return e;
    }
    const dim3 g(T / RB, nt);
    auto kw = RB == 8 ? bitmask_w_kernel<8> : (RB == 4 ? bitmask_w_kernel<4> : bitmask_w_kernel<2>);
    return launch_kernel(kw, g, kMaskThreads, smem, s, nullptr, I.W, I.s, region, counts, member,
                         K, T, bitmask);
  }
  const int RB = mask_rows(K);
  const size_t smem = (size_t)RB * (((size_t)K + 7) & ~size_t(7)) * sizeof(float) + (size_t)K;
  for (const void* fn : {(const void*)bitmask_kernel<1>, (const void*)bitmask_kernel<2>,
                         (const void*)bitmask_kernel<4>, (const void*)bitmask_kernel<8>}) {
    e = set_max_dynamic_smem(fn, 96 * 1024 + kMaxK);
    if (e != cudaSuccess) return e;
  }
  const dim3 g(T / RB, nt);
  auto ki = RB == 8 ? bitmask_kernel<8>
                    : (RB == 4 ? bitmask_kernel<4> : (RB == 2 ? bitmask_kernel<2> : bitmask_kernel<1>));
  return launch_kernel(ki, g, kMaskThreads, smem, s, nullptr, I, region, counts, member, K, T,
                       bitmask);
}

}  // namespace hinm
