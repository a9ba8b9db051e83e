// a4. Mask: regions by rank, 2:4 groups in ascending working position, top-2 of 4 per
// row (FlexHiNM-GP notes, 亮点与洞察: high -> dense, middle -> 2:4, low -> pruned;
// rkmt.cn section 二: keep 2 of every 4 consecutive; geek-doc.cn section 五: the mask has
// W's shape).
//
//   inverse_perm_kernel   pinv[perm[j]] = j (checks that perm is a permutation)
//   classify_kernel       one CTA per tile: region of every working position and the
//                         2:4 members in ascending working position (member[t][q])
//   bitmask_kernel        one CTA per (tile, 16 rows): dense words by ballot over the
//                         region, 2:4 groups top-2 of 4 per row, words assembled in shared
//                         memory and written once, coalesced.
#include <cuda_runtime.h>

#include "hinm_internal.h"
#include "ptx.cuh"

namespace hinm {

// pinv must be preset to -1.  A repeated or out-of-range channel is reported as
// HINM_ERR_INVALID_ARG (the permutation is then not a permutation of 0..K-1).
__global__ void inverse_perm_kernel(const int32_t* __restrict__ perm, int K,
                                    int32_t* __restrict__ pinv, int* status) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const int c = perm ? __ldg(perm + j) : j;
  if (c < 0 || c >= K) {
    ptx::record_status(status, HINM_ERR_INVALID_ARG);
    return;
  }
  if (atomicExch(pinv + c, j) != -1) ptx::record_status(status, HINM_ERR_INVALID_ARG);
}

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
                                                        const int32_t* __restrict__ perm,
                                                        const int32_t* __restrict__ counts, int K,
                                                        int8_t* __restrict__ region,
                                                        int32_t* __restrict__ member,
                                                        int* status) {
  __shared__ int warp_tot[32];
  __shared__ int total;
  const int t = blockIdx.x;
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
      mem[pos++] = j;
    }
    reg[c] = cls;
  }
}

// One CTA per (tile, kMaskRows rows): the rows' mask words are assembled in shared memory.
// Dense bits are the same in every row of the tile (one ballot per word over the region
// array); each 2:4 group is handled by one thread for all the CTA's rows.
constexpr int kMaskRows = 16;

__global__ void __launch_bounds__(256) bitmask_kernel(
    const float* __restrict__ I, const int32_t* __restrict__ perm,
    const int8_t* __restrict__ region, const int32_t* __restrict__ counts,
    const int32_t* __restrict__ member, int M, int K, int T, uint32_t* __restrict__ bitmask) {
  extern __shared__ uint32_t words_s[];  // [kMaskRows][words]
  const int words = (K + 31) >> 5;
  const int t = blockIdx.y;
  const int r0 = blockIdx.x * kMaskRows;  // first row of the chunk within the tile
  const int rows = min(kMaskRows, T - r0);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  const int8_t* reg = region + (size_t)t * K;

  // dense bits: warp per word, lane = bit
  for (int w = warp; w < words; w += nwarps) {
    const int c = w * 32 + lane;
    const bool dense = c < K && __ldg(reg + c) == HINM_REGION_DENSE;
    const uint32_t bits = __ballot_sync(0xffffffffu, dense);
    if (lane < rows) words_s[lane * words + w] = bits;
  }
  __syncthreads();

  int n24 = counts[3 * t + 1];
  const int n0 = counts[3 * t], n4 = counts[3 * t + 2];
  if (n0 < 0 || n24 < 0 || n4 < 0 || n0 + n24 + n4 != K || (n24 & 3)) n24 = 0;
  const int ng = n24 / 4;
  const int32_t* mem = member + (size_t)t * K;
  const float* I0 = I + ((size_t)t * T + r0) * K;
  for (int g = threadIdx.x; g < ng; g += blockDim.x) {
    int c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      int j = __ldg(mem + 4 * g + k);
      j = ((unsigned)j < (unsigned)K) ? j : 0;  // never index outside perm / I
      c[k] = ptx::perm_at(perm, j, K);
    }
    const float* row = I0;
#pragma unroll 4
    for (int r = 0; r < rows; ++r, row += K) {
      float v[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) v[k] = __ldg(row + c[k]);
      // beats[k]: members ranked above k (greater value, or equal value at a lower position)
      int beats[4] = {0, 0, 0, 0};
#pragma unroll
      for (int k = 0; k < 4; ++k)
#pragma unroll
        for (int l = k + 1; l < 4; ++l) {
          if (v[l] > v[k]) ++beats[k];
          else ++beats[l];  // v[k] >= v[l]: k (lower position) ranks above l
        }
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (beats[k] < 2) atomicOr(words_s + r * words + (c[k] >> 5), 1u << (c[k] & 31));
    }
  }
  __syncthreads();
  uint32_t* out = bitmask + ((size_t)t * T + r0) * words;
  for (int x = threadIdx.x; x < rows * words; x += blockDim.x) out[x] = words_s[x];
}

size_t mask_workspace_bytes(int M, int K, int T) {
  const int nt = M / T;
  Carve c{nullptr, 0};
  c.take<double>((size_t)nt * K);   // V (only when no rank is passed)
  c.take<int32_t>((size_t)nt * K);  // rank (only when no rank is passed)
  c.take<int32_t>((size_t)K);       // inverse permutation
  c.take<int32_t>((size_t)nt * K);  // member
  c.take<int>((size_t)nt);          // tile max exponent (by-product of the ranking)
  c.take<char>(rank_scratch_bytes(M, K, T));
  return (c.off + 255) & ~size_t(255);
}

cudaError_t launch_mask(const float* I, const int32_t* perm, const int32_t* counts,
                        const int32_t* rank, int M, int K, int T, uint32_t* bitmask,
                        int8_t* region, void* ws, int* status, cudaStream_t s) {
  const int nt = M / T;
  Carve cv{static_cast<char*>(ws), 0};
  double* V = cv.take<double>((size_t)nt * K);
  int32_t* rank_ws = cv.take<int32_t>((size_t)nt * K);
  int32_t* pinv = cv.take<int32_t>((size_t)K);
  int32_t* member = cv.take<int32_t>((size_t)nt * K);
  int* pmax = cv.take<int>((size_t)nt);
  char* rank_scratch = cv.take<char>(rank_scratch_bytes(M, K, T));
  cudaError_t e;
  if (!rank) {
    e = launch_vector_rank(I, perm, M, K, T, V, rank_ws, pmax, rank_scratch, s);
    if (e != cudaSuccess) return e;
    rank = rank_ws;
  }
  e = cudaMemsetAsync(pinv, 0xFF, (size_t)K * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  inverse_perm_kernel<<<(K + 255) / 256, 256, 0, s>>>(perm, K, pinv, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  classify_kernel<<<nt, 1024, 0, s>>>(rank, perm, counts, K, region, member, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int words = (K + 31) / 32;
  const size_t smem = (size_t)kMaskRows * words * sizeof(uint32_t);
  static bool attr_set = false;
  if (!attr_set) {
    e = cudaFuncSetAttribute(bitmask_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)(kMaskRows * ((kMaxK + 31) / 32) * sizeof(uint32_t)));
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 g((T + kMaskRows - 1) / kMaskRows, nt);
  bitmask_kernel<<<g, 256, smem, s>>>(I, perm, region, counts, member, M, K, T, bitmask);
  return cudaGetLastError();
}

}  // namespace hinm
