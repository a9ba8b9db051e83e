// a5. Compress W ⊙ M into the HiNM layout (FlexHiNM-GP notes, 关键设计 2/4: dense part and
// 2:4 part stored apart, the 2:4 part gathered by a precomputed index with the input
// permutation folded in; geek-doc.cn section 三: 2 values per group plus 2-bit positions).
//
//   tile_info_kernel   per tile: dense blocks ceil(n4/64), sparse blocks ceil(n24/128),
//                      prefix offsets; checks counts and buffer capacity
//   lists_kernel       per tile: dense and 2:4 working positions in ascending order
//   pack_kernel        one CTA per (block, tile): writes one 16 KB value block exactly as
//                      the tensor cores read it from shared memory (128-byte swizzle),
//                      the 2 KB metadata block in tensor-memory lane order, and the index.
#include <cuda_runtime.h>

#include "hinm_internal.h"
#include "ptx.cuh"

namespace hinm {

// One CTA of 1024 threads: each thread takes a contiguous run of tiles; the block offsets
// are an exclusive prefix sum over the tiles.  Should the blocks exceed the layout's
// capacity (the caller sized it for other counts), the tiles are walked in order instead,
// and a tile that does not fit gets no blocks.
constexpr int kTileInfoThreads = 1024;

__device__ __forceinline__ void tile_blocks(const int32_t* counts, int t, int K, int& nd, int& ns,
                                            int* status) {
  const int n0 = counts[3 * t], n24 = counts[3 * t + 1], n4 = counts[3 * t + 2];
  nd = ns = 0;
  if (n0 < 0 || n24 < 0 || n4 < 0 || n0 + n24 + n4 != K || (n24 & 3)) {
    ptx::record_status(status, HINM_ERR_INVALID_ARG);
  } else {
    nd = (n4 + kDenseBK - 1) / kDenseBK;
    ns = (n24 + kSparseBK - 1) / kSparseBK;
  }
}

__global__ void __launch_bounds__(kTileInfoThreads) tile_info_kernel(
    const int32_t* __restrict__ counts, int nt, int K, int max_dense, int max_sparse,
    int32_t* __restrict__ info, int* status) {
  __shared__ int wd[32], ws[32];
  __shared__ int tot_d, tot_s;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int per = (nt + kTileInfoThreads - 1) / kTileInfoThreads;
  const int t0 = threadIdx.x * per, t1 = min(nt, t0 + per);
  int sd = 0, ss = 0;
  for (int t = t0; t < t1; ++t) {
    int nd, ns;
    tile_blocks(counts, t, K, nd, ns, nullptr);
    sd += nd;
    ss += ns;
  }
  // exclusive block scan of (sd, ss)
  int id = sd, is = ss;
  for (int o = 1; o < 32; o <<= 1) {
    const int xd = __shfl_up_sync(0xffffffffu, id, o), xs = __shfl_up_sync(0xffffffffu, is, o);
    if (lane >= o) {
      id += xd;
      is += xs;
    }
  }
  if (lane == 31) {
    wd[warp] = id;
    ws[warp] = is;
  }
  __syncthreads();
  if (warp == 0) {
    const int vd = wd[lane], vs = ws[lane];
    int cd = vd, cs = vs;
    for (int o = 1; o < 32; o <<= 1) {
      const int xd = __shfl_up_sync(0xffffffffu, cd, o), xs = __shfl_up_sync(0xffffffffu, cs, o);
      if (lane >= o) {
        cd += xd;
        cs += xs;
      }
    }
    wd[lane] = cd - vd;
    ws[lane] = cs - vs;
    if (lane == 31) {
      tot_d = cd;
      tot_s = cs;
    }
  }
  __syncthreads();
  if (tot_d <= max_dense && tot_s <= max_sparse) {
    int d0 = wd[warp] + id - sd, s0 = ws[warp] + is - ss;
    for (int t = t0; t < t1; ++t) {
      int nd, ns;
      tile_blocks(counts, t, K, nd, ns, status);
      info[4 * t + 0] = nd;
      info[4 * t + 1] = ns;
      info[4 * t + 2] = d0;
      info[4 * t + 3] = s0;
      d0 += nd;
      s0 += ns;
    }
    return;
  }
  if (threadIdx.x != 0) return;
  int d0 = 0, s0 = 0;
  for (int t = 0; t < nt; ++t) {
    int nd, ns;
    tile_blocks(counts, t, K, nd, ns, status);
    if (d0 + nd > max_dense || s0 + ns > max_sparse) {
      ptx::record_status(status, HINM_ERR_WORKSPACE);
      nd = ns = 0;
    }
    info[4 * t + 0] = nd;
    info[4 * t + 1] = ns;
    info[4 * t + 2] = d0;
    info[4 * t + 3] = s0;
    d0 += nd;
    s0 += ns;
  }
}

// lists[t][0 .. n_dense) = dense working positions, lists[t][n_dense .. ) = 2:4 ones.
__global__ void __launch_bounds__(1024) lists_kernel(const int8_t* __restrict__ region,
                                                     const int32_t* __restrict__ perm_all,
                                                     long long perm_stride,
                                                     const int32_t* __restrict__ counts, int K,
                                                     int32_t* __restrict__ lists, int* status) {
  __shared__ int warp_tot[2][32];
  const int t = blockIdx.x;
  const int32_t* perm = perm_all ? perm_all + t * perm_stride : perm_all;  // this tile's order
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int8_t* reg = region + (size_t)t * K;
  const int per = (K + blockDim.x - 1) / blockDim.x;
  const int j0 = threadIdx.x * per, j1 = min(K, j0 + per);
  int cd = 0, cs = 0;
  for (int j = j0; j < j1; ++j) {
    const int8_t r = reg[ptx::perm_at(perm, j, K)];
    cd += (r == HINM_REGION_DENSE);
    cs += (r == HINM_REGION_24);
  }
  int id = cd, is = cs;
  for (int o = 1; o < 32; o <<= 1) {
    const int a = __shfl_up_sync(0xffffffffu, id, o), b = __shfl_up_sync(0xffffffffu, is, o);
    if (lane >= o) {
      id += a;
      is += b;
    }
  }
  if (lane == 31) {
    warp_tot[0][warp] = id;
    warp_tot[1][warp] = is;
  }
  __syncthreads();
  int bd = 0, bs = 0, td = 0, ts = 0;
  for (int w = 0; w < nw; ++w) {
    if (w < warp) {
      bd += warp_tot[0][w];
      bs += warp_tot[1][w];
    }
    td += warp_tot[0][w];
    ts += warp_tot[1][w];
  }
  const int n4 = counts[3 * t + 2], n24 = counts[3 * t + 1];
  if (threadIdx.x == 0 && (td != n4 || ts != n24)) ptx::record_status(status, HINM_ERR_INVALID_ARG);
  int pd = bd + id - cd, ps = td + bs + is - cs;
  int32_t* L = lists + (size_t)t * K;
  for (int j = j0; j < j1; ++j) {
    const int8_t r = reg[ptx::perm_at(perm, j, K)];
    if (r == HINM_REGION_DENSE) L[pd++] = j;
    else if (r == HINM_REGION_24) L[ps++] = j;
  }
}

__device__ __forceinline__ int swz(int r, int k) {  // byte offset of bf16 (r, k) in a block
  return r * 128 + ((((k >> 3) ^ (r & 7))) << 4) + (k & 7) * 2;
}

// Working position stored in a list entry, clamped into [0, K) so that inconsistent
// region / counts arguments (reported in the status word) never index out of bounds.
__device__ __forceinline__ int list_at(const int32_t* lst, int p, int K) {
  const int j = lst[p];
  return (unsigned)j < (unsigned)K ? j : 0;
}

__device__ __forceinline__ bool mask_bit(const uint32_t* bm, int words, int i, int c) {
  return (__ldg(bm + (size_t)i * words + (c >> 5)) >> (c & 31)) & 1u;
}

// A malformed group (not exactly two kept positions) is reported (HINM_ERR_BAD_MASK); its
// kept positions, lowest first, are completed from the unkept ones with value 0, so the pair
// stays a legal (a < b) pattern.  Out of line: it is rare, and inlined into every unrolled
// item it would crowd the packing loops out of the instruction cache.
__device__ __noinline__ void select_pair_malformed(uint32_t w0, uint32_t w1, uint32_t w2,
                                                   uint32_t w3, uint32_t kept, uint32_t* out,
                                                   int* status) {
  const uint32_t w[4] = {w0, w1, w2, w3};
  ptx::record_status(status, HINM_ERR_BAD_MASK);
  int pos[2], np = 0;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (((kept >> k) & 1u) && np < 2) pos[np++] = k;
#pragma unroll
  for (int k = 0; k < 4; ++k)
    if (!((kept >> k) & 1u) && np < 2) pos[np++] = -1 - k;  // filler, value 0
  const int pa = pos[0] < 0 ? -1 - pos[0] : pos[0];
  const int pb = pos[1] < 0 ? -1 - pos[1] : pos[1];
  const bool ua = pos[0] >= 0, ub = pos[1] >= 0;
  if (pa < pb) {  // order the pair by position
    out[0] = pa; out[1] = pb; out[2] = ua ? w[pa] : 0u; out[3] = ub ? w[pb] : 0u;
  } else {
    out[0] = pb; out[1] = pa; out[2] = ub ? w[pb] : 0u; out[3] = ua ? w[pa] : 0u;
  }
}

// The stored pair of one 2:4 group from its 4 weights and kept bits: positions a < b and
// their values.  The common case has exactly two kept positions.
__device__ __forceinline__ void select_pair(const uint32_t (&w)[4], uint32_t kept, uint32_t& a,
                                            uint32_t& bb, uint32_t& va, uint32_t& vb,
                                            int* status) {
  if (__popc(kept) == 2) {
    a = (uint32_t)(__ffs(kept) - 1);
    bb = (uint32_t)(31 - __clz(kept));
    va = a == 0 ? w[0] : (a == 1 ? w[1] : w[2]);   // a <= 2
    vb = bb == 1 ? w[1] : (bb == 2 ? w[2] : w[3]);  // b >= 1
    return;
  }
  uint32_t out[4];
  select_pair_malformed(w[0], w[1], w[2], w[3], kept, out, status);
  a = out[0];
  bb = out[1];
  va = out[2];
  vb = out[3];
}

__global__ void __launch_bounds__(256) pack_kernel(const uint16_t* __restrict__ W,
                                                   const uint32_t* __restrict__ bitmask,
                                                   const int32_t* __restrict__ perm_all,
                                                   long long perm_stride,
                                                   const int32_t* __restrict__ counts,
                                                   const int32_t* __restrict__ lists, int K, int T,
                                                   hinm_layout L, int* status) {
  __shared__ uint8_t nib[128][32];
  __shared__ int chan[kSparseBK];  // input channel of every vector of the block, -1 = padding
  const int t = blockIdx.y;
  const int b = blockIdx.x;
  const int32_t* perm = perm_all ? perm_all + t * perm_stride : perm_all;  // this tile's order
  const int nd = L.tile_info[4 * t + 0], ns = L.tile_info[4 * t + 1];
  const int d0 = L.tile_info[4 * t + 2], s0 = L.tile_info[4 * t + 3];
  if (b >= nd + ns) return;
  const int n4 = counts[3 * t + 2], n24 = counts[3 * t + 1];
  const int words = (K + 31) >> 5;
  const int32_t* lst = lists + (size_t)t * K;
  const int row0 = t * T;
  const bool sparse = b >= nd;
  const int sb = b - nd;
  const int nvec = sparse ? kSparseBK : kDenseBK;
  if (threadIdx.x < nvec) {
    const int p = sparse ? sb * kSparseBK + threadIdx.x : b * kDenseBK + threadIdx.x;
    const int lim = sparse ? n24 : n4;
    chan[threadIdx.x] = p < lim ? ptx::perm_at(perm, list_at(lst, (sparse ? n4 : 0) + p, K), K) : -1;
  }
  __syncthreads();
  // index and contiguous-run flag
  if (threadIdx.x < nvec) {
    const int v = chan[threadIdx.x] < 0 ? 0 : chan[threadIdx.x];
    if (sparse) L.idx_sparse[(size_t)(s0 + sb) * kSparseBK + threadIdx.x] = v;
    else L.idx_dense[(size_t)(d0 + b) * kDenseBK + threadIdx.x] = v;
  }
  const int c0 = chan[0] < 0 ? 0 : chan[0];
  const bool step_ok = threadIdx.x >= nvec || chan[threadIdx.x] == c0 + (int)threadIdx.x;
  const bool run = __syncthreads_and(step_ok);
  if (threadIdx.x == 0) {
    if (sparse) L.run_sparse[s0 + sb] = run ? c0 : -1;
    else L.run_dense[d0 + b] = run ? c0 : -1;
  }

  // a block whose channels are one run c0, c0+1, ...: a group's (or 8 vectors') weights are
  // consecutive in W's row and their mask bits share one word, so they move with one load each
  const bool run8 = run && (c0 & 7) == 0 && (K & 7) == 0;  // 16-byte loads of 8 weights
  const bool run4 = run && (c0 & 3) == 0;                  // 8-byte loads of 4 weights

  if (!sparse) {
    uint8_t* out = reinterpret_cast<uint8_t*>(L.vals_dense + (size_t)(d0 + b) * 8192);
#pragma unroll 2
    for (int item = threadIdx.x; item < 128 * 8; item += blockDim.x) {
      const int r = item >> 3, ch = item & 7;
      uint32_t h[8];
      if (r < T && run8) {
        const int i = row0 + r;
        const int cb = c0 + ch * 8;
        const uint4 wv = __ldg(reinterpret_cast<const uint4*>(W + (size_t)i * K + cb));
        const uint32_t bits = (__ldg(bitmask + (size_t)i * words + (cb >> 5)) >> (cb & 31)) & 0xFFu;
        const uint32_t wr[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          h[2 * p] = ((bits >> (2 * p)) & 1u) ? (wr[p] & 0xFFFFu) : 0u;
          h[2 * p + 1] = ((bits >> (2 * p + 1)) & 1u) ? (wr[p] >> 16) : 0u;
        }
      } else if (r < T) {
        const int i = row0 + r;
        const uint16_t* Wi = W + (size_t)i * K;
        const uint32_t* bmi = bitmask + (size_t)i * words;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int c = chan[ch * 8 + e];
          const int cc = c < 0 ? 0 : c;
          const uint32_t w = __ldg(Wi + cc);
          const uint32_t bit = (__ldg(bmi + (cc >> 5)) >> (cc & 31)) & 1u;
          h[e] = (c >= 0 && bit) ? w : 0u;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) h[e] = 0u;
      }
      uint4 q;
      q.x = h[0] | (h[1] << 16);
      q.y = h[2] | (h[3] << 16);
      q.z = h[4] | (h[5] << 16);
      q.w = h[6] | (h[7] << 16);
      *reinterpret_cast<uint4*>(out + r * 128 + ((ch ^ (r & 7)) << 4)) = q;
    }
    return;
  }

  uint8_t* out = reinterpret_cast<uint8_t*>(L.vals_sparse + (size_t)(s0 + sb) * 8192);
  if (run4) {
    // contiguous run: per thread, the loads of kU items go out before any is processed
    constexpr int kU = 4;
    for (int base = threadIdx.x; base < 128 * 32; base += 256 * kU) {
      uint2 wv[kU];
      uint32_t mw[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int item = base + 256 * u;
        const int r = min(item >> 5, T - 1), g = item & 31;  // rows >= T: any valid row, unused
        const int cb = c0 + 4 * g;
        wv[u] = __ldg(reinterpret_cast<const uint2*>(W + (size_t)(row0 + r) * K + cb));
        mw[u] = __ldg(bitmask + (size_t)(row0 + r) * words + (cb >> 5));
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int item = base + 256 * u;
        const int r = item >> 5, g = item & 31;
        uint32_t a = 0, bb = 1, va = 0, vb = 0;
        if (r < T) {
          const uint32_t w[4] = {wv[u].x & 0xFFFFu, wv[u].x >> 16, wv[u].y & 0xFFFFu,
                                 wv[u].y >> 16};
          select_pair(w, (mw[u] >> ((c0 + 4 * g) & 31)) & 0xFu, a, bb, va, vb, status);
        }
        *reinterpret_cast<uint32_t*>(out + swz(r, 2 * g)) = va | (vb << 16);
        nib[r][g] = (uint8_t)(a | (bb << 2));
      }
    }
  } else {
#pragma unroll 4
    for (int item = threadIdx.x; item < 128 * 32; item += blockDim.x) {
      const int r = item >> 5, g = item & 31;
      uint32_t a = 0, bb = 1, va = 0, vb = 0;
      if (r < T && chan[4 * g] >= 0) {
        const int i = row0 + r;
        const uint16_t* Wi = W + (size_t)i * K;
        const uint32_t* bmi = bitmask + (size_t)i * words;
        uint32_t w[4], kept = 0;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int c = chan[4 * g + k];
          w[k] = __ldg(Wi + c);
          kept |= ((__ldg(bmi + (c >> 5)) >> (c & 31)) & 1u) << k;
        }
        select_pair(w, kept, a, bb, va, vb, status);
      }
      *reinterpret_cast<uint32_t*>(out + swz(r, 2 * g)) = va | (vb << 16);
      nib[r][g] = (uint8_t)(a | (bb << 2));
    }
  }
  __syncthreads();
  uint32_t* meta = L.meta + (size_t)(s0 + sb) * kMetaWords;
  for (int wi = threadIdx.x; wi < kMetaWords; wi += blockDim.x) {
    const int lane = wi >> 2, w = wi & 3;
    const int h = (lane >> 3) & 1;
    uint32_t word = 0;
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const int m = 16 * (lane >> 4) + 8 * s + (lane & 7);
#pragma unroll
      for (int q = 0; q < 4; ++q) word |= uint32_t(nib[m][8 * w + 4 * h + q]) << (16 * s + 4 * q);
    }
    meta[wi] = word;
  }
}

size_t compress_workspace_bytes(int M, int K, int T) {
  const int nt = M / T;
  return (((size_t)nt * K * sizeof(int32_t)) + 255) & ~size_t(255);
}

// Cross-layer index translation, one CTA per (block, tile) as pack_kernel: every index
// entry c of the block becomes row_of_channel[c], then the block's run flag is recomputed
// (first index when the entries are one ascending run, else -1).  An entry or map value
// outside [0, K) is reported as HINM_ERR_INVALID_ARG and written as 0.
__global__ void __launch_bounds__(kSparseBK) translate_index_kernel(
    const int32_t* __restrict__ row_of_channel, int K, hinm_layout L, int* status) {
  __shared__ int first;
  const int t = blockIdx.y, b = blockIdx.x;
  const int nd = L.tile_info[4 * t + 0], ns = L.tile_info[4 * t + 1];
  if (b >= nd + ns) return;
  const bool sparse = b >= nd;
  const int nvec = sparse ? kSparseBK : kDenseBK;
  const int blk = sparse ? L.tile_info[4 * t + 3] + b - nd : L.tile_info[4 * t + 2] + b;
  if (blk < 0 || blk >= (sparse ? L.max_sparse_blocks : L.max_dense_blocks)) {
    // tile_info not from hinm_compress for this layout: report, touch nothing
    if (threadIdx.x == 0) ptx::record_status(status, HINM_ERR_INVALID_ARG);
    return;
  }
  int32_t* idx = sparse ? L.idx_sparse + (size_t)blk * kSparseBK : L.idx_dense + (size_t)blk * kDenseBK;
  int v = 0;
  if ((int)threadIdx.x < nvec) {
    const int c = idx[threadIdx.x];
    if (c >= 0 && c < K) v = __ldg(row_of_channel + c);
    if (c < 0 || c >= K || v < 0 || v >= K) {
      ptx::record_status(status, HINM_ERR_INVALID_ARG);
      v = 0;
    }
    idx[threadIdx.x] = v;
  }
  if (threadIdx.x == 0) first = v;
  __syncthreads();
  const bool step_ok = (int)threadIdx.x >= nvec || v == first + (int)threadIdx.x;
  const bool run = __syncthreads_and(step_ok);
  if (threadIdx.x == 0) (sparse ? L.run_sparse : L.run_dense)[blk] = run ? first : -1;
}

cudaError_t launch_translate_index(const hinm_layout& L, const int32_t* row_of_channel,
                                   int* status, cudaStream_t s) {
  const int nt = L.num_tiles, K = L.K;
  if (nt <= 0) return cudaSuccess;
  const int max_blocks = (K + kDenseBK - 1) / kDenseBK + (K + kSparseBK - 1) / kSparseBK;
  translate_index_kernel<<<dim3(max_blocks, nt), kSparseBK, 0, s>>>(row_of_channel, K, L, status);
  return cudaGetLastError();
}

cudaError_t launch_compress(const uint16_t* W, const uint32_t* bitmask, const int8_t* region,
                            const int32_t* perm, long long perm_stride, const int32_t* counts,
                            int M, int K, int T,
                            const hinm_layout& L, void* ws, int* status, cudaStream_t s) {
  const int nt = M / T;
  int32_t* lists = static_cast<int32_t*>(ws);
  tile_info_kernel<<<1, kTileInfoThreads, 0, s>>>(counts, nt, K, L.max_dense_blocks,
                                                  L.max_sparse_blocks, L.tile_info, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // lists are read only at positions below the counts, so no clearing is needed
  lists_kernel<<<nt, 1024, 0, s>>>(region, perm, perm_stride, counts, K, lists, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int max_blocks = (K + kDenseBK - 1) / kDenseBK + (K + kSparseBK - 1) / kSparseBK;
  dim3 g(max_blocks, nt);
  pack_kernel<<<g, 256, 0, s>>>(W, bitmask, perm, perm_stride, counts, lists, K, T, L, status);
  return cudaGetLastError();
}

}  // namespace hinm
