// a4. Mask: regions by rank, 2:4 groups in ascending working position, top-2 of 4 per
// row (FlexHiNM-GP notes, 亮点与洞察: high -> dense, middle -> 2:4, low -> pruned;
// rkmt.cn section 二: keep 2 of every 4 consecutive; geek-doc.cn section 五: the mask has
// W's shape).
//
//   inverse_perm_kernel   pinv[perm[j]] = j
//   classify_kernel       one CTA per tile: region of every working position, prefix
//                         count of the 2:4 vectors -> pos24[t][j] and member[t][q]
//   bitmask_kernel        one warp per 32-channel word of a row: dense -> 1, pruned -> 0,
//                         2:4 -> top-2 of the group's 4 importances; __ballot_sync packs
//                         the word, so every word is written once, coalesced.
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
                                                        int32_t* __restrict__ pos24,
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
  int32_t* p24 = pos24 + (size_t)t * K;
  int32_t* mem = member + (size_t)t * K;
  for (int j = j0; j < j1; ++j) {
    const int r = rk[j];
    const int c = ptx::perm_at(perm, j, K);
    int8_t cls = HINM_REGION_PRUNED;
    if (r < n4) {
      cls = HINM_REGION_DENSE;
      p24[j] = -1;
    } else if (r < n4 + n24) {
      cls = HINM_REGION_24;
      mem[pos] = j;
      p24[j] = pos++;
    } else {
      p24[j] = -1;
    }
    reg[c] = cls;
  }
}

__global__ void bitmask_kernel(const float* __restrict__ I, const int32_t* __restrict__ perm,
                               const int32_t* __restrict__ pinv, const int8_t* __restrict__ region,
                               const int32_t* __restrict__ pos24, const int32_t* __restrict__ member,
                               int M, int K, int T, uint32_t* __restrict__ bitmask) {
  const int words = (K + 31) >> 5;
  const int w = blockIdx.y * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int i = blockIdx.x;
  const int lane = threadIdx.x & 31;
  if (w >= words) return;
  const int t = i / T;
  const int c = w * 32 + lane;
  bool keep = false;
  if (c < K) {
    const int8_t reg = __ldg(region + (size_t)t * K + c);
    if (reg == HINM_REGION_DENSE) {
      keep = true;
    } else if (reg == HINM_REGION_24) {
      const int j = __ldg(pinv + c);
      const int p = ((unsigned)j < (unsigned)K) ? __ldg(pos24 + (size_t)t * K + j) : -1;
      if (p >= 0) {
        const int g = p >> 2, slot = p & 3;
        const float* Ii = I + (size_t)i * K;
        const int32_t* mem = member + (size_t)t * K + 4 * g;
        const float v = __ldg(Ii + c);
        int beats = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          if (k == slot) continue;
          int jk = __ldg(mem + k);
          jk = ((unsigned)jk < (unsigned)K) ? jk : 0;  // never index outside perm / I
          const int ck = ptx::perm_at(perm, jk, K);
          const float vk = __ldg(Ii + ck);
          beats += (vk > v) || (vk == v && k < slot);
        }
        keep = beats < 2;
      }
    }
  }
  const unsigned word = __ballot_sync(0xffffffffu, keep);
  if (lane == 0) bitmask[(size_t)i * words + w] = word;
}

size_t mask_workspace_bytes(int M, int K, int T) {
  const int nt = M / T;
  Carve c{nullptr, 0};
  c.take<double>((size_t)nt * K);   // V (only when no rank is passed)
  c.take<int32_t>((size_t)nt * K);  // rank (only when no rank is passed)
  c.take<int32_t>((size_t)K);       // inverse permutation
  c.take<int32_t>((size_t)nt * K);  // pos24
  c.take<int32_t>((size_t)nt * K);  // member
  c.take<int>((size_t)nt);          // tile max exponent (by-product of the ranking)
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
  int32_t* pos24 = cv.take<int32_t>((size_t)nt * K);
  int32_t* member = cv.take<int32_t>((size_t)nt * K);
  int* pmax = cv.take<int>((size_t)nt);
  cudaError_t e;
  if (!rank) {
    e = launch_vector_rank(I, perm, M, K, T, V, rank_ws, pmax, s);
    if (e != cudaSuccess) return e;
    rank = rank_ws;
  }
  e = cudaMemsetAsync(pinv, 0xFF, (size_t)K * sizeof(int32_t), s);
  if (e != cudaSuccess) return e;
  inverse_perm_kernel<<<(K + 255) / 256, 256, 0, s>>>(perm, K, pinv, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  classify_kernel<<<nt, 1024, 0, s>>>(rank, perm, counts, K, region, pos24, member, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int words = (K + 31) / 32;
  dim3 g(M, (words + 7) / 8);
  bitmask_kernel<<<g, 256, 0, s>>>(I, perm, pinv, region, pos24, member, M, K, T, bitmask);
  return cudaGetLastError();
}

}  // namespace hinm
