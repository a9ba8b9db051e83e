// a5. Compress W ⊙ M into the HiNM layout (FlexHiNM-GP notes, 关键设计 2/4: dense part and
// 2:4 part stored apart, the 2:4 part gathered by a precomputed index with the input
// permutation folded in; geek-doc.cn section 三: 2 values per group plus 2-bit positions).
//
//   tile_info_kernel   per tile: dense blocks ceil(n4/64), sparse blocks ceil(n24/128),
//                      prefix offsets; checks counts and buffer capacity
//   slots_kernel       per tile: the channel of every vector slot of its blocks (padding
//                      marked), the working order folded in
//   pack_rows_kernel   (K <= 8192) one CTA per (chunk of block rows, tile): the rows of W
//                      and of the mask staged in shared memory, the blocks written from
//                      there; pack_kernel (K > 8192) one CTA per (block, tile), gathering
//                      from L2.  Both write every 16 KB value block exactly as the tensor
//                      cores read it from shared memory (128-byte swizzle), the 2 KB
//                      metadata block in tensor-memory lane order, and the index.
#include <cuda_runtime.h>

#include "hinm_internal.h"
#include "launch.cuh"
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
  ptx::enter_dependent();
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

// The tile's block slots: slots[t][s] = the input channel of vector slot s of the tile's
// blocks, kNoChan for padding.  Slots [0, nd*64) are the dense blocks' (dense channels in
// ascending working position, then padding), slots [nd*64, nd*64 + ns*128) the 2:4 blocks'
// (the 2:4 channels likewise), nd = ceil(n4/64), ns = ceil(n24/128) from the counts.  The
// tile's working order is folded in here, once.  Every entry of the row is written (padding
// first), and writes stay inside the row whatever the region and counts arguments hold
// (a mismatch between them is reported in the status word), so the packing reads only
// kNoChan or channels below K.
constexpr uint16_t kNoChan = 0xFFFFu;

__host__ __device__ inline size_t slot_stride(int K) {  // uint16 entries per tile, 16-byte rows
  return ((size_t)K + 192 + 7) & ~size_t(7);           // nd*64 + ns*128 <= K + 190
}

__global__ void __launch_bounds__(1024) slots_kernel(const int8_t* __restrict__ region,
                                                     const int32_t* __restrict__ perm_all,
                                                     long long perm_stride,
                                                     const int32_t* __restrict__ counts, int K,
                                                     uint16_t* __restrict__ slots, int* status) {
  ptx::enter_dependent();
  __shared__ int warp_tot[2][32];
  const int t = blockIdx.x;
  const int32_t* perm = perm_all ? perm_all + t * perm_stride : perm_all;  // this tile's order
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int8_t* reg = region + (size_t)t * K;
  const int S = (int)slot_stride(K);
  uint16_t* row = slots + (size_t)t * S;
  for (int p = threadIdx.x; p < S; p += blockDim.x) row[p] = kNoChan;
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
  __syncthreads();  // also orders the padding fill before the channel writes
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
  const int sparse0 = (n4 >= 0 && n4 <= K) ? (n4 + kDenseBK - 1) / kDenseBK * kDenseBK : 0;
  int pd = bd + id - cd, ps = sparse0 + bs + is - cs;
  for (int j = j0; j < j1; ++j) {
    const int c = ptx::perm_at(perm, j, K);
    const int8_t r = reg[c];
    if (r == HINM_REGION_DENSE) {
      if (pd < sparse0) row[pd] = (uint16_t)c;
      ++pd;
    } else if (r == HINM_REGION_24) {
      if (ps < S) row[ps] = (uint16_t)c;
      ++ps;
    }
  }
}

__device__ __forceinline__ int swz(int r, int k) {  // byte offset of bf16 (r, k) in a block
  return r * 128 + ((((k >> 3) ^ (r & 7))) << 4) + (k & 7) * 2;
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
                                                   const uint16_t* __restrict__ slots, int K,
                                                   int T, hinm_layout L, int* status) {
  ptx::enter_dependent();
  __shared__ uint8_t nib[128][32];
  __shared__ int chan[kSparseBK];  // input channel of every vector of the block, -1 = padding
  const int t = blockIdx.y;
  const int b = blockIdx.x;
  const int nd = L.tile_info[4 * t + 0], ns = L.tile_info[4 * t + 1];
  const int d0 = L.tile_info[4 * t + 2], s0 = L.tile_info[4 * t + 3];
  if (b >= nd + ns) return;
  const int words = (K + 31) >> 5;
  const uint16_t* slt = slots + (size_t)t * slot_stride(K);
  const int row0 = t * T;
  const bool sparse = b >= nd;
  const int sb = b - nd;
  const int nvec = sparse ? kSparseBK : kDenseBK;
  if (threadIdx.x < nvec) {
    const int p = sparse ? nd * kDenseBK + sb * kSparseBK + threadIdx.x : b * kDenseBK + threadIdx.x;
    const uint16_t c = p < (int)slot_stride(K) ? slt[p] : kNoChan;
    chan[threadIdx.x] = c == kNoChan ? -1 : (int)c;
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

// Row-staged packing: one CTA of 16 warps per (chunk of R block rows, tile).  The tile's
// slot -> channel map (kNoChan = padding) and the chunk's rows of W and of the bitmask are
// copied into shared memory with cp.async (every row read once, coalesced), then the chunk's
// (block, row) items are dealt to the warps in contiguous block-major ranges, so a warp loads
// a block's channels, and works out their shared-memory offsets, once for several rows.  A
// dense block row is 64 channels (2 per lane), a sparse block row 32 groups (one per lane);
// each leaves as one 128-byte line, and a sparse row's metadata as 16-bit halves (rows m and
// m + 8 share each word).  The channel gathers hit shared memory, not L2.  Rows past T
// (T = 64) load nothing and are written as zero values with the padding pair (positions 0
// and 1), as every padded group is.  R is chosen so that two CTAs fit an SM.
struct PackSmem {
  size_t chan, ring, row_w, row_bm, stage, total;
};

__host__ __device__ inline PackSmem pack_smem(int K, int rows) {
  PackSmem p;
  p.chan = 0;
  p.ring = slot_stride(K) * 2;
  p.row_w = ((size_t)K * 2 + 15) & ~size_t(15);
  p.row_bm = (((size_t)K + 31) / 32 * 4 + 15) & ~size_t(15);
  p.stage = p.row_w + p.row_bm;
  p.total = p.ring + (size_t)rows * p.stage;
  return p;
}

using ptx::cp_async16;
using ptx::cp_async4;
using ptx::cp_async8;
using ptx::cp_async_commit_wait_all;

constexpr int kPackThreads = 512;
constexpr int kPackWarps = kPackThreads / 32;

__global__ void __launch_bounds__(kPackThreads, 2) pack_rows_kernel(
    const uint16_t* __restrict__ W, const uint32_t* __restrict__ bitmask,
    const uint16_t* __restrict__ slots, int K, int T, int R, hinm_layout L, int* status) {
  ptx::enter_dependent();
  extern __shared__ __align__(16) uint8_t sm[];
  const PackSmem lay = pack_smem(K, R);
  const uint16_t* chan = reinterpret_cast<const uint16_t*>(sm + lay.chan);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = blockIdx.y;
  const int m0 = blockIdx.x * R;                      // first block row of the chunk
  const int rc = min(R, kSparseBK - m0);              // rows in this chunk
  const int live_rows = max(0, min(rc, T - m0));      // of which inside the tile
  const int nd = L.tile_info[4 * t + 0], ns = L.tile_info[4 * t + 1];
  const int d0 = L.tile_info[4 * t + 2], s0 = L.tile_info[4 * t + 3];
  const int nslot_d = nd * kDenseBK, nslot = nslot_d + ns * kSparseBK;
  if (nd + ns == 0 || rc <= 0) return;
  if (nd < 0 || ns < 0 || nd > (K + kDenseBK - 1) / kDenseBK ||
      ns > (K + kSparseBK - 1) / kSparseBK || nslot > (int)slot_stride(K)) {  // other counts
    if (threadIdx.x == 0) ptx::record_status(status, HINM_ERR_INVALID_ARG);
    return;
  }
  const int words = (K + 31) >> 5;
  {  // the tile's slot map and the chunk's rows, one copy group
    const uint16_t* src = slots + (size_t)t * slot_stride(K);
    const uint32_t dst = ptx::smem_u32(sm + lay.chan);
    for (int q = threadIdx.x; q < (nslot + 7) / 8; q += kPackThreads)
      cp_async16(dst + 16 * q, src + 8 * q);
    const uint32_t ring = ptx::smem_u32(sm + lay.ring);
    for (int a = 0; a < live_rows; ++a) {
      const uint32_t rd = ring + (uint32_t)(a * lay.stage);
      const uint16_t* wsrc = W + (size_t)(t * T + m0 + a) * K;
      if ((K & 7) == 0) {
        for (int q = threadIdx.x; q < (K >> 3); q += kPackThreads) cp_async16(rd + 16 * q, wsrc + 8 * q);
      } else {
        for (int q = threadIdx.x; q < (K >> 2); q += kPackThreads) cp_async8(rd + 8 * q, wsrc + 4 * q);
      }
      const uint32_t* bsrc = bitmask + (size_t)(t * T + m0 + a) * words;
      const uint32_t bd = rd + (uint32_t)lay.row_w;
      for (int q = threadIdx.x; q < words; q += kPackThreads) cp_async4(bd + 4 * q, bsrc + q);
    }
    cp_async_commit_wait_all();
    __syncthreads();
  }
  if (blockIdx.x == 0) {  // the index and the contiguous-run flag of every block of the tile
    for (int b = warp; b < nd + ns; b += kPackWarps) {
      const bool sparse = b >= nd;
      const int base = sparse ? nslot_d + (b - nd) * kSparseBK : b * kDenseBK;
      const int per = sparse ? kSparseBK / 32 : kDenseBK / 32;
      const int cf = chan[base] == kNoChan ? 0 : chan[base];
      bool ok = true;
      for (int e = lane * per; e < (lane + 1) * per; ++e) {
        const int c = chan[base + e];
        ok = ok && c != kNoChan && c == cf + e;
        const int v = c == kNoChan ? 0 : c;
        if (sparse) L.idx_sparse[(size_t)(s0 + b - nd) * kSparseBK + e] = v;
        else L.idx_dense[(size_t)(d0 + b) * kDenseBK + e] = v;
      }
      const bool run = __all_sync(0xffffffffu, ok);
      if (lane == 0) {
        if (sparse) L.run_sparse[s0 + b - nd] = run ? cf : -1;
        else L.run_dense[d0 + b] = run ? cf : -1;
      }
    }
  }

  // this warp's contiguous range of (block, row) items, block-major
  const int n = (nd + ns) * rc;
  const int i0 = (int)((long long)n * warp / kPackWarps);
  const int i1 = (int)((long long)n * (warp + 1) / kPackWarps);
  if (i0 >= i1) return;
  int b = i0 / rc, a = i0 - (i0 / rc) * rc;
  int cur = -1;
  uint32_t c[4] = {kNoChan, kNoChan, kNoChan, kNoChan};  // this lane's channels of block b
  uint8_t* out = nullptr;
  uint16_t* meta = nullptr;
  bool run = false;  // block b's channels are one aligned run: vector loads from the row
  const int hw = lane >> 3, hh = (lane >> 2) & 1;  // (w, h) of the lane's metadata half
  for (int i = i0; i < i1; ++i) {
    const bool sparse = b >= nd;
    if (b != cur) {  // warp-uniform: a new block
      cur = b;
      if (!sparse) {
        const uint32_t cc = *reinterpret_cast<const uint32_t*>(chan + b * kDenseBK + 2 * lane);
        c[0] = cc & 0xFFFFu;
        c[1] = cc >> 16;
        const uint32_t base = __shfl_sync(0xffffffffu, c[0], 0);
        run = __all_sync(0xffffffffu, (base & 1u) == 0 && c[0] == base + 2 * lane &&
                                          c[1] == c[0] + 1);
        out = reinterpret_cast<uint8_t*>(L.vals_dense + (size_t)(d0 + b) * 8192);
      } else {
        const uint2 cv = *reinterpret_cast<const uint2*>(chan + nslot_d + (b - nd) * kSparseBK +
                                                         4 * lane);
        c[0] = cv.x & 0xFFFFu;
        c[1] = cv.x >> 16;
        c[2] = cv.y & 0xFFFFu;
        c[3] = cv.y >> 16;
        const uint32_t base = __shfl_sync(0xffffffffu, c[0], 0);
        run = __all_sync(0xffffffffu, (base & 3u) == 0 && c[0] == base + 4 * lane &&
                                          c[1] == c[0] + 1 && c[2] == c[0] + 2 && c[3] == c[0] + 3);
        // a group is whole or all padding; with region and counts arguments that disagree
        // (reported by slots_kernel) a member may be missing: read channel 0 in its place
#pragma unroll
        for (int k = 1; k < 4; ++k) c[k] = c[k] == kNoChan ? 0u : c[k];
        out = reinterpret_cast<uint8_t*>(L.vals_sparse + (size_t)(s0 + b - nd) * 8192);
        meta = reinterpret_cast<uint16_t*>(L.meta + (size_t)(s0 + b - nd) * kMetaWords);
      }
    }
    const int m = m0 + a;  // row within the block
    const bool live = a < live_rows;
    const uint8_t* stage = sm + lay.ring + (size_t)a * lay.stage;
    const uint16_t* wrow = reinterpret_cast<const uint16_t*>(stage);
    const uint32_t* brow = reinterpret_cast<const uint32_t*>(stage + lay.row_w);
    const int off = swz(m, 2 * lane);
    if (!sparse) {
      uint32_t h[2] = {0u, 0u};
      if (run) {  // channels c[0], c[0] + 1 (even): one 4-byte load, their bits in one word
        if (live) {
          const uint32_t wv = *reinterpret_cast<const uint32_t*>(wrow + c[0]);
          const uint32_t bits = brow[c[0] >> 5] >> (c[0] & 31);
          h[0] = (bits & 1u) ? (wv & 0xFFFFu) : 0u;
          h[1] = (bits & 2u) ? (wv >> 16) : 0u;
        }
      } else {
#pragma unroll
        for (int k = 0; k < 2; ++k)
          h[k] = (live && c[k] != kNoChan && ((brow[c[k] >> 5] >> (c[k] & 31)) & 1u))
                     ? (uint32_t)wrow[c[k]] : 0u;
      }
      *reinterpret_cast<uint32_t*>(out + off) = h[0] | (h[1] << 16);
    } else {
      uint32_t pa = 0, pb = 1, va = 0, vb = 0;
      if (live && c[0] != kNoChan) {
        uint32_t w[4], kept = 0;
        if (run) {  // channels c[0] .. c[0] + 3 (c[0] a multiple of 4): one 8-byte load
          const uint2 wv = *reinterpret_cast<const uint2*>(wrow + c[0]);
          w[0] = wv.x & 0xFFFFu;
          w[1] = wv.x >> 16;
          w[2] = wv.y & 0xFFFFu;
          w[3] = wv.y >> 16;
          kept = (brow[c[0] >> 5] >> (c[0] & 31)) & 0xFu;
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            w[k] = wrow[c[k]];
            kept |= ((brow[c[k] >> 5] >> (c[k] & 31)) & 1u) << k;
          }
        }
        select_pair(w, kept, pa, pb, va, vb, status);
      }
      *reinterpret_cast<uint32_t*>(out + off) = va | (vb << 16);
      // group g = 8w + 4h + q: the 4 nibbles of (w, h) form one half of a metadata word
      uint32_t x = (pa | (pb << 2)) << (4 * (lane & 3));
      x |= __shfl_xor_sync(0xffffffffu, x, 1);
      x |= __shfl_xor_sync(0xffffffffu, x, 2);
      if ((lane & 3) == 0)  // half (m / 8) mod 2 of word w of lane 16 (m / 16) + 8 h + m mod 8
        meta[2 * (4 * (16 * (m >> 4) + 8 * hh + (m & 7)) + hw) + ((m >> 3) & 1)] = (uint16_t)x;
    }
    if (++a == rc) {
      a = 0;
      ++b;
    }
  }
}

// Rows per CTA for pack_rows_kernel: up to 8, fewer while two CTAs would not fit an SM.
inline int pack_rows_per_cta(int K) {
  int R = 8;
  while (R > 1 && pack_smem(K, R).total > 113 * 1024) --R;
  return R;
}

size_t compress_workspace_bytes(int M, int K, int T) {
  const int nt = M / T;
  return (((size_t)nt * slot_stride(K) * sizeof(uint16_t)) + 255) & ~size_t(255);
}

// Cross-layer index translation, one CTA per (block, tile) as pack_kernel: every index
// entry c of the block becomes row_of_channel[c], then the block's run flag is recomputed
// (first index when the entries are one ascending run, else -1).  An entry or map value
// outside [0, K) is reported as HINM_ERR_INVALID_ARG and written as 0.
__global__ void __launch_bounds__(kSparseBK) translate_index_kernel(
    const int32_t* __restrict__ row_of_channel, int K, hinm_layout L, int* status) {
  ptx::enter_dependent();
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
  return launch_kernel(translate_index_kernel, dim3(max_blocks, nt), kSparseBK, 0, s, nullptr,
                       row_of_channel, K, L, status);
}

cudaError_t launch_compress(const uint16_t* W, const uint32_t* bitmask, const int8_t* region,
                            const int32_t* perm, long long perm_stride, const int32_t* counts,
                            int M, int K, int T,
                            const hinm_layout& L, void* ws, int* status, cudaStream_t s) {
  const int nt = M / T;
  uint16_t* slots = static_cast<uint16_t*>(ws);
  cudaError_t e = launch_kernel(tile_info_kernel, 1, kTileInfoThreads, 0, s, nullptr, counts, nt,
                                K, L.max_dense_blocks, L.max_sparse_blocks, L.tile_info, status);
  if (e != cudaSuccess) return e;
  e = launch_kernel(slots_kernel, nt, 1024, 0, s, nullptr, region, perm, perm_stride, counts, K,
                    slots, status);
  if (e != cudaSuccess) return e;
  // Long rows (K > 8192) leave room for fewer rows per CTA than the staging needs to pay
  // off; there one CTA per (block, tile) gathers from L2 (measured on B200, K = 11008:
  // 71-73 us against 73-91 us for the row-staged kernel; K = 4096 with a random order:
  // 90 us against 66 us).
  if (K > 8192) {
    const int max_blocks = (K + kDenseBK - 1) / kDenseBK + (K + kSparseBK - 1) / kSparseBK;
    dim3 g(max_blocks, nt);
    return launch_kernel(pack_kernel, g, 256, 0, s, nullptr, W, bitmask, slots, K, T, L, status);
  }
  const int R = pack_rows_per_cta(K);
  const size_t smem = pack_smem(K, R).total;
  e = set_max_dynamic_smem((const void*)pack_rows_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 g((kSparseBK + R - 1) / R, nt);  // every block row, also those past T
  return launch_kernel(pack_rows_kernel, g, kPackThreads, smem, s, nullptr, W, bitmask, slots, K,
                       T, R, L, status);
}

}  // namespace hinm
