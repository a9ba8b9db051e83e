// a6. HiNM SpMM on the sm_100a tensor cores (FlexHiNM-GP notes, 关键设计 4: the dense part
// and the 2:4 part, the latter gathered by the precomputed index, summed into one output).
//
// The pages run two CUDA streams (mma and mma.sp) merged by atomicAdd.  Here a persistent
// kernel (one CTA per SM) walks work units (tile, BN-column block); in each unit both kinds
// of K-block accumulate into ONE tensor-memory accumulator, double-buffered so the
// epilogue of a unit overlaps the main loop of the next.  At narrow N, when the units fill
// less than half of the SMs, a cluster of up to 8 CTAs shares each unit's K-blocks and the
// leader adds the others' partial accumulators (received over DSMEM) in rank order.
//
// Warp roles (G = 8 gather warps in the persistent kernel at BN >= 128, else 4):
//   warps 0..G-1  gather producers: for a K-block whose index is not one contiguous run,
//              the X rows it selects, 16-byte cp.async into the swizzled MN-major B tile
//              (coalesced 2*BN-byte row segments); arrival on the stage's barrier when
//              they land.
//   warp G     MMA: one thread; 2:4 block -> tcgen05.cp of the metadata into tensor memory,
//              then 4 x tcgen05.mma.sp (K = 32 each); dense block -> 4 x tcgen05.mma
//              (K = 16 each); tcgen05.commit frees the stage / publishes the accumulator.
//   warps G+1..G+4  epilogue: tcgen05.ld of the 128 x BN fp32 accumulator (a lane holds one
//              row; warp w reads lane quadrant w mod 4), 32 columns at a time transposed
//              through a per-warp swizzled 4 KB shared tile so that each store instruction
//              writes 128-byte row segments of four rows of Y (or, in a split-K cluster, to
//              the leader's reduction buffer).
//   warp G+5   bulk copies: one thread runs ahead by up to a full ring; per K-block it
//              publishes the block's run flag and index list and bulk-copies the
//              pre-swizzled 16 KB A block, its 2 KB metadata and, for a contiguous run,
//              the X rows as 3-D tiled TMA boxes (one per 64 K-rows).
//
// spmm_pair_kernel (T = 128, wide N, on the caller's hint that tiles select the same X rows)
// takes tile pairs x 240 columns with the same roles: where both tiles' blocks are the same
// runs of X rows, one B stage feeds the MMAs of both tiles (two accumulators in tensor
// memory), else the pair's tiles run one after the other.
//
// Shared memory holds STAGES stages of [A 16 KB | B 128 x BN bf16 | E 2 KB]; the stage ring
// runs across work units.  At wide N the second 64 K-rows of a stage complete a barrier of
// their own, so that the first two MMAs of a 2:4 block do not wait for them.  Every load
// brings data to its own CTA only.  Every wait is bounded (2 s), after which the CTA records
// HINM_ERR_DEVICE_TIMEOUT, stops all roles, drains what it issued, frees tensor memory and
// returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "hinm_internal.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace hinm {

template <int BN, bool SPLIT = false>
struct SpmmCfg {
  static constexpr int kAtom = BN >= 64 ? 64 : BN;  // B swizzle atom width (elements)
  static constexpr int kAtomBytes = kAtom * 2;      // 128, 64 or 32 bytes
  static constexpr int kSwzBits = kAtomBytes == 128 ? 3 : (kAtomBytes == 64 ? 2 : 1);
  static constexpr int kChunksPerAtom = kAtomBytes / 16;
  static constexpr int kChunksPerRow = BN / 8;
  static constexpr int kABytes = kBlockBytes;
  // B tile: two halves of 64 K-rows (a 2:4 block uses both, a dense block the first); each
  // half holds its column atoms one after another, 64 rows x kAtomBytes each
  static constexpr int kBHalfBytes = 64 * BN * 2;
  static constexpr int kBBytes = 2 * kBHalfBytes;
  static constexpr int kBAtomStride = 64 * kAtomBytes;
  static constexpr int kEBytes = 2048;
  // a stage is a multiple of 1024 bytes (the 128-byte swizzle atoms stay aligned); each
  // stage's vector indices (gathered blocks) live in a separate region after the stages
  static constexpr int kStageBytes = kABytes + kBBytes + kEBytes;
  static constexpr int kIdxBytes = 512;
  // split-K: CTAs of a cluster per unit; the leader's reduction buffer holds the others'
  // 128 x BN fp32 partial accumulators
  static constexpr int kMaxSplit = !SPLIT ? 1 : (BN <= 16 ? 8 : 4);
  static constexpr int kRedBytes = (kMaxSplit - 1) * 128 * BN * 4;
  static constexpr int kStagesRaw = (210 * 1024 - kRedBytes) / (kStageBytes + kIdxBytes);
  static constexpr int kStages = kStagesRaw > 8 ? 8 : kStagesRaw;
  // layout type of the B descriptor: 2 = 128-byte swizzle, 4 = 64-byte, 6 = 32-byte
  static constexpr uint32_t kBLayout = kAtomBytes == 128 ? 2u : (kAtomBytes == 64 ? 4u : 6u);
  static constexpr int kAccCols = BN < 32 ? 32 : BN;  // accumulator buffer stride (columns)
  // two accumulator buffers (epilogue overlaps the next unit) when tensor memory holds them
  static constexpr int kAccBufs = 2 * kAccCols + 4 * kStages <= 512 ? 2 : 1;
  static constexpr int kTmemNeed = kAccBufs * kAccCols + 4 * kStages;
  static constexpr int kTmemCols = kTmemNeed <= 32 ? 32 : kTmemNeed <= 64 ? 64 : kTmemNeed <= 128 ? 128
                                   : kTmemNeed <= 256 ? 256 : 512;
  // persistent kernel with 32-column chunks: one 32 x 32 fp32 staging tile per epilogue
  // warp, through which its lanes' accumulator rows become 128-byte row segments of Y
  static constexpr int kEpiBytes = (SPLIT || BN < 32) ? 0 : 4 * 32 * 32 * 4;
  static constexpr size_t kSmemBytes = (size_t)kStages * (kStageBytes + kIdxBytes) +
                                       1024 /*align*/ + 512 /*barriers*/ + kRedBytes + kEpiBytes;
  // wide N: the second 64 K-rows of a 2:4 block's B land on a barrier of their own, so the
  // MMAs on the first 64 rows start before the second half arrives
  static constexpr bool kSplitB = BN >= 128;
  // 8 gather warps for the persistent kernel at BN >= 128 (more 16-byte copies in flight:
  // measured 2 % faster on the up-proj and gate shapes than 4), else 4; then one MMA warp,
  // 4 epilogue warps and one bulk-copy warp
  static constexpr int kProducers = (!SPLIT && BN >= 128) ? 256 : 128;
  static constexpr int kMmaWarp = kProducers / 32;
  static constexpr int kBulkWarp = kMmaWarp + 5;
  static constexpr int kThreads = kProducers + 192;
  static_assert(BN == 16 || BN == 32 || (BN % 64 == 0 && BN <= 256), "BN");
  static_assert(kStages >= 2, "stages");
  static_assert(kTmemNeed <= 512, "tmem");
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(!SPLIT || BN <= 32, "split-K is for narrow N");
};

struct SpmmArgs {
  const int32_t* tile_info;
  const uint16_t* vals_dense;
  const uint16_t* vals_sparse;
  const uint32_t* meta;
  const int32_t* idx_dense;
  const int32_t* idx_sparse;
  const int32_t* run_dense;
  const int32_t* run_sparse;
  const uint16_t* X;
  float* Y;
  int N, T;
  int num_tiles, nblk_n, num_units;
  int split;  // CTAs (one cluster) per unit; 1 = persistent, no split
  int x3d;    // the X tensor map is 3-D (columns within an atom, rows, atoms)
  int* status;
  // epilogue: y = act(acc + bias[row]), stored as fp32 to Y or, when Yb is set, as bf16 to Yb
  const float* bias;  // per output row, or nullptr
  int act;            // HINM_ACT_*
  uint16_t* Yb;
};

__device__ __forceinline__ float epi_act(float x, int act) {
  if (act == HINM_ACT_RELU) return fmaxf(x, 0.0f);
  if (act == HINM_ACT_SILU) return __fdiv_rn(x, __fadd_rn(1.0f, expf(-x)));
  if (act == HINM_ACT_GELU)
    return __fmul_rn(__fmul_rn(0.5f, x), __fadd_rn(1.0f, erff(__fmul_rn(x, 0.70710678118654752f))));
  return x;
}
// v[0..n): fp32 bits of one row's accumulator columns -> act(v + b)
template <int NV>
__device__ __forceinline__ void epi_apply(uint32_t (&v)[32], float b, int act) {
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = __float_as_uint(epi_act(__fadd_rn(__uint_as_float(v[i]), b), act));
}
// bf16 (round to nearest even) of two fp32 bit patterns, packed low | high << 16
__device__ __forceinline__ uint32_t pack_bf16x2(uint32_t lo, uint32_t hi) {
  const __nv_bfloat162 h = __float22bfloat162_rn(make_float2(__uint_as_float(lo), __uint_as_float(hi)));
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// X rows idx[0..ROWS) (columns n0 .. n0+BN) -> the swizzled MN-major B tile, 16 bytes per
// cp.async; consecutive threads copy consecutive 16-byte pieces of a row (coalesced).
template <class C, int ROWS>
struct Gather {
  static constexpr int kPer = ROWS * C::kChunksPerRow / C::kProducers;
  static_assert(kPer * C::kProducers == ROWS * C::kChunksPerRow, "chunks per producer");
  int xr[kPer];
  // the block's indices, brought into the stage by the bulk-copy warp
  __device__ __forceinline__ void load_index(const int* idx_s, int ptid) {
#pragma unroll
    for (int i = 0; i < kPer; ++i) xr[i] = idx_s[(ptid + C::kProducers * i) / C::kChunksPerRow];
  }
  // items [I0, I1): item i covers row (ptid + kProducers i) / kChunksPerRow, so for 128 rows
  // the first kPer / 2 items are rows 0..63 and the rest rows 64..127
  template <int I0 = 0, int I1 = kPer>
  __device__ __forceinline__ void copy(uint32_t B_s, const uint16_t* __restrict__ X, int N,
                                       int n0, int ptid) const {
#pragma unroll
    for (int i = I0; i < I1; ++i) {
      const int q = ptid + C::kProducers * i;
      const int r = q / C::kChunksPerRow, cc = q - r * C::kChunksPerRow;
      const int at = cc / C::kChunksPerAtom, c = cc - at * C::kChunksPerAtom;
      const int col = n0 + cc * 8;
      const bool ok = col < N;
      const uint16_t* src = ok ? X + (size_t)xr[i] * N + col : X;
      uint32_t off = (r >> 6) * C::kBHalfBytes + at * C::kBAtomStride + (r & 63) * C::kAtomBytes +
                     c * 16;
      off ^= ((off >> 7) & ((1u << C::kSwzBits) - 1u)) << 4;  // shared-memory swizzle
      cp_async_16(B_s + off, src, ok ? 16u : 0u);
    }
  }
};

// One warp's 32 rows x cw (<= 32, a multiple of 8) columns of Y: lane l holds row r0 + l's
// values v.  They go through the warp's swizzled 4 KB shared tile (16-byte pieces, piece
// slot XOR row mod 8) and out as row segments: 128 bytes of 4 rows per fp32 store
// instruction, 64 bytes of 8 rows per bf16 one.  rows are tile rows (rows >= T not stored).
__device__ __forceinline__ void store_chunk32(const SpmmArgs& a, uint32_t ep, uint32_t (&v)[32],
                                              int lane, int r0, int tile, int gc0, int cw) {
  if (a.Yb) {
    uint32_t h[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) h[j] = pack_bf16x2(v[2 * j], v[2 * j + 1]);
#pragma unroll
    for (int p = 0; p < 4; ++p)
      ptx::st_shared_v4(ep + lane * 128 + ((p ^ (lane & 7)) << 4), h[4 * p], h[4 * p + 1],
                        h[4 * p + 2], h[4 * p + 3]);
    __syncwarp();
    const int rr = lane >> 2, pc = lane & 3;
    const int gc = gc0 + 8 * pc;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int r = 8 * i + rr;
      const uint4 o = ptx::ld_shared_v4(ep + r * 128 + ((pc ^ (r & 7)) << 4));
      const int rw = r0 + r;
      if (8 * pc < cw && rw < a.T)
        *reinterpret_cast<uint4*>(a.Yb + (size_t)(tile * a.T + rw) * a.N + gc) = o;
    }
  } else {
#pragma unroll
    for (int p = 0; p < 8; ++p)
      ptx::st_shared_v4(ep + lane * 128 + ((p ^ (lane & 7)) << 4), v[4 * p], v[4 * p + 1],
                        v[4 * p + 2], v[4 * p + 3]);
    __syncwarp();
    const int rr = lane >> 3, pc = lane & 7;
    const int gc = gc0 + 4 * pc;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int r = 4 * i + rr;
      const uint4 o = ptx::ld_shared_v4(ep + r * 128 + ((pc ^ (r & 7)) << 4));
      const int rw = r0 + r;
      if (4 * pc < cw && rw < a.T)
        *reinterpret_cast<uint4*>(a.Y + (size_t)(tile * a.T + rw) * a.N + gc) = o;
    }
  }
  __syncwarp();  // the tile is rewritten by the next chunk
}

// One row's n (16 or 32) columns from column gc: fp32 or bf16, 16-byte stores while the row
// has room for them (N % 8 == 0), else element by element.
__device__ __forceinline__ void store_row(const SpmmArgs& a, const uint32_t (&v)[32], int n,
                                          int grow, int gc) {
  if (a.Yb) {
    uint16_t* yr = a.Yb + (size_t)grow * a.N;
    for (int i = 0; i < n; i += 8) {
      if (gc + i + 8 <= a.N) {
        *reinterpret_cast<uint4*>(yr + gc + i) =
            make_uint4(pack_bf16x2(v[i], v[i + 1]), pack_bf16x2(v[i + 2], v[i + 3]),
                       pack_bf16x2(v[i + 4], v[i + 5]), pack_bf16x2(v[i + 6], v[i + 7]));
      }
    }
  } else {
    float* yr = a.Y + (size_t)grow * a.N;
    for (int i = 0; i < n; i += 4) {
      if (gc + i + 4 <= a.N)
        *reinterpret_cast<float4*>(yr + gc + i) =
            make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                        __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]));
    }
  }
}

template <int BN, bool SPLIT>
__global__ void __launch_bounds__(SpmmCfg<BN, SPLIT>::kThreads, 1)
    spmm_kernel(const __grid_constant__ CUtensorMap tmX, const SpmmArgs a) {
  using C = SpmmCfg<BN, SPLIT>;
  extern __shared__ uint8_t smem_raw[];
  ptx::enter_dependent();
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* idx_region = smem + C::kStages * C::kStageBytes;  // [S][kIdxBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(idx_region + C::kStages * C::kIdxBytes);
  // [0,S) full, [S,2S) empty, 2S+{0,1} accumulator full, 2S+{2,3} accumulator empty,
  // 2S+4 drain, [2S+5, 3S+5) index ready, [3S+5, 4S+5) second-half full; then the TMEM
  // address, the abort flag and one run flag per stage (at most 336 bytes of the 512 reserved)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * C::kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* run_s = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return ptx::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return ptx::smem_u32(bars + C::kStages + s); };
  auto accf_bar = [&](int b) { return ptx::smem_u32(bars + 2 * C::kStages + b); };
  auto acce_bar = [&](int b) { return ptx::smem_u32(bars + 2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = ptx::smem_u32(bars + 2 * C::kStages + 4);
  auto idx_bar = [&](int s) { return ptx::smem_u32(bars + 2 * C::kStages + 5 + s); };
  auto full2_bar = [&](int s) { return ptx::smem_u32(bars + 3 * C::kStages + 5 + s); };

  // Work: persistent CTAs stride over the units; split-K CTAs take one unit each and the
  // K-block range [kb0, kb1) of their cluster rank.
  const int u_first = SPLIT ? (int)blockIdx.x / a.split : (int)blockIdx.x;
  const int u_step = SPLIT ? a.num_units : (int)gridDim.x;
  const int rank = SPLIT ? (int)(blockIdx.x % a.split) : 0;
  auto k_range = [&](int nblk, int& kb0, int& kb1) {
    kb0 = SPLIT ? (int)((long long)nblk * rank / a.split) : 0;
    kb1 = SPLIT ? (int)((long long)nblk * (rank + 1) / a.split) : nblk;
  };
  // Run flag of K-block kb of a tile with record info (the bulk-copy warp's lanes load 32
  // consecutive blocks' flags at once).
  auto run_flag = [&](const int4& info, int kb) {
    const bool sparse = kb >= info.x;
    const size_t blk = sparse ? (size_t)(info.w + kb - info.x) : (size_t)(info.z + kb);
    return __ldg(sparse ? a.run_sparse + blk : a.run_dense + blk);
  };
  // The first unit's tile record, and for the bulk-copy warp the run flags of its first 32
  // K-blocks (one per lane), are loaded before the set-up below, so that their latency
  // overlaps it.
  int4 info_first = make_int4(0, 0, 0, 0);
  int run_first = -1;
  if (u_first < a.num_units) {
    info_first = __ldg(reinterpret_cast<const int4*>(a.tile_info) + u_first / a.nblk_n);
    if (warp == C::kBulkWarp) {
      int kb0, kb1;
      k_range(info_first.x + info_first.y, kb0, kb1);
      if (kb0 + lane < kb1) run_first = run_flag(info_first, kb0 + lane);
    }
  }
  auto tile_info_of = [&](int u, int tile) {
    return u == u_first ? info_first : __ldg(reinterpret_cast<const int4*>(a.tile_info) + tile);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(full_bar(s), 1 + C::kProducers);  // expect_tx arrival + one per producer
      ptx::mbar_init(empty_bar(s), 1);
      ptx::mbar_init(idx_bar(s), 1);
      ptx::mbar_init(full2_bar(s), 1 + C::kProducers);  // used when kSplitB
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(accf_bar(b), 1);
      ptx::mbar_init(acce_bar(b), 4);  // one arrival per epilogue warp
    }
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == C::kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t meta_col0 = C::kAccBufs * C::kAccCols;
  float* red = reinterpret_cast<float*>(idx_region + C::kStages * C::kIdxBytes + 512);
  // [4 warps][32 rows][8 x 16-byte pieces], piece p of row r at slot p ^ (r & 7)
  uint8_t* epi_stage = reinterpret_cast<uint8_t*>(red) + C::kRedBytes;

  // split-K: what the leader's epilogue needs after the cluster barrier
  bool split_ready = false, split_has = false;
  int split_tile = 0, split_n0 = 0, split_b = 0;

  if (warp < C::kProducers / 32) {
    // ------------------------------------------------------------ gather producers
    // Per K-block: wait until the bulk-copy warp has the stage (its index-ready barrier),
    // then either gather the X rows the block's index selects (16-byte cp.async, arrival
    // when they land) or, for a contiguous run it moves by TMA, just arrive.  Every thread
    // arrives on the stage's full barrier once per block, after its last read of the
    // stage's run flag and indices, so the stage cannot be recycled under it.  With
    // kSplitB, rows 64..127 of a 2:4 block arrive on the stage's second-half barrier (every
    // thread arrives there once per block too, after its first-half arrival).
    const int ptid = threadIdx.x;
    uint32_t it = 0;  // K-blocks handled by this CTA (stage ring position)
    bool stop = false;
    for (int u = u_first; u < a.num_units && !stop; u += u_step) {
      const int tile = u / a.nblk_n, n0 = (u - tile * a.nblk_n) * BN;
      const int4 info = tile_info_of(u, tile);
      const int nd = info.x, nblk = info.x + info.y;
      int kb0, kb1;
      k_range(nblk, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
        const bool sparse = kb >= nd;
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (!ptx::mbar_wait(idx_bar(s), ph, a.status, abort_flag)) {
          stop = true;
          break;
        }
        const int run = run_s[s];
        const uint32_t A_s = ptx::smem_u32(smem + s * C::kStageBytes);
        const uint32_t B_s = A_s + C::kABytes;
        const int* idx_s = reinterpret_cast<const int*>(idx_region + s * C::kIdxBytes);
        if (run < 0) {
          if (sparse) {
            using G = Gather<C, kSparseBK>;
            G gs;
            gs.load_index(idx_s, ptid);
            if constexpr (C::kSplitB) {
              gs.template copy<0, G::kPer / 2>(B_s, a.X, a.N, n0, ptid);
              cp_async_arrive_noinc(full_bar(s));
              gs.template copy<G::kPer / 2, G::kPer>(B_s, a.X, a.N, n0, ptid);
              cp_async_arrive_noinc(full2_bar(s));
            } else {
              gs.copy(B_s, a.X, a.N, n0, ptid);
              cp_async_arrive_noinc(full_bar(s));
            }
          } else {
            Gather<C, kDenseBK> gd;
            gd.load_index(idx_s, ptid);
            gd.copy(B_s, a.X, a.N, n0, ptid);
            cp_async_arrive_noinc(full_bar(s));
            if constexpr (C::kSplitB) ptx::mbar_arrive(full2_bar(s));
          }
        } else {
          ptx::mbar_arrive(full_bar(s));
          if constexpr (C::kSplitB) ptx::mbar_arrive(full2_bar(s));
        }
      }
    }
    cp_async_wait_all();
  } else if (warp == C::kBulkWarp) {
    // ------------------------------------------------------------ bulk copies
    // One thread runs ahead of the gather warps by up to a full ring: per K-block, once the
    // stage is free, it publishes the block's run flag and index list (index-ready barrier)
    // and bulk-copies the pre-swizzled A block, its metadata and, for a contiguous run, the
    // X rows by TMA (full barrier).  The warp's lanes load the run flags of 32 blocks at a
    // time, so the issuing thread does not wait for one global load per block (with few
    // MMAs per stage, as at N = 16, that wait bounded the rate at which stages refilled).
    uint32_t it = 0;
    bool stop = false;
    for (int u = u_first; u < a.num_units && !stop; u += u_step) {
      const int tile = u / a.nblk_n, n0 = (u - tile * a.nblk_n) * BN;
      const int4 info = tile_info_of(u, tile);
      const int nd = info.x, nblk = info.x + info.y;
      int kb0, kb1;
      k_range(nblk, kb0, kb1);
      for (int base = kb0; base < kb1 && !stop; base += 32) {
        int run_l = -1;
        if (u == u_first && base == kb0)
          run_l = run_first;
        else if (base + lane < kb1)
          run_l = run_flag(info, base + lane);
        const int nb = min(32, kb1 - base);
        for (int q = 0; q < nb; ++q, ++it) {
          const int run = __shfl_sync(0xffffffffu, run_l, q);
          int ok = 1;
          if (lane == 0) {
            const int kb = base + q;
            const bool sparse = kb >= nd;
            const size_t blk = sparse ? (size_t)(info.w + kb - nd) : (size_t)(info.z + kb);
            const int s = it % C::kStages;
            const uint32_t ph = (it / C::kStages) & 1;
            ok = ptx::mbar_wait(empty_bar(s), ph ^ 1, a.status, abort_flag) ? 1 : 0;
            if (ok) {
              const uint32_t A_s = ptx::smem_u32(smem + s * C::kStageBytes);
              const uint32_t B_s = A_s + C::kABytes;
              const uint32_t E_s = B_s + C::kBBytes;
              const uint32_t I_s = ptx::smem_u32(idx_region + s * C::kIdxBytes);
              const int rows = sparse ? kSparseBK : kDenseBK;
              run_s[s] = run;  // published by the arrive below (release)
              if (run < 0) {
                ptx::mbar_arrive_expect_tx(idx_bar(s), (uint32_t)rows * 4u);
                ptx::bulk_g2s(I_s, sparse ? a.idx_sparse + blk * kSparseBK : a.idx_dense + blk * kDenseBK,
                              (uint32_t)rows * 4u, idx_bar(s));
              } else {
                ptx::mbar_arrive(idx_bar(s));
              }
              // with kSplitB the full barrier takes A, metadata and the first 64 rows of X; the
              // second-half barrier the rest of a run's rows (none for a dense block or a gather)
              const int rows1 = C::kSplitB ? 64 : rows;
              const uint32_t bytes = C::kABytes + (sparse ? C::kEBytes : 0) +
                                     (run >= 0 ? (uint32_t)rows1 * BN * 2u : 0u);
              ptx::mbar_arrive_expect_tx(full_bar(s), bytes);
              if constexpr (C::kSplitB)
                ptx::mbar_arrive_expect_tx(full2_bar(s),
                                           run >= 0 ? (uint32_t)(rows - rows1) * BN * 2u : 0u);
              ptx::bulk_g2s(A_s, (sparse ? a.vals_sparse : a.vals_dense) + blk * 8192, C::kABytes,
                            full_bar(s));
              if (sparse) ptx::bulk_g2s(E_s, a.meta + blk * kMetaWords, C::kEBytes, full_bar(s));
              if (run >= 0) {
                // one ascending run of X rows: per half of 64 rows, one 3-D box over all the
                // column atoms, or one 2-D box per atom
#pragma unroll 1
                for (int h = 0; h < rows / 64; ++h) {
                  const uint32_t fb = (C::kSplitB && h == 1) ? full2_bar(s) : full_bar(s);
                  if (a.x3d) {
                    ptx::tma_load_3d(B_s + h * C::kBHalfBytes, &tmX, 0, run + h * 64, n0 / C::kAtom,
                                     fb);
                  } else {
#pragma unroll 1
                    for (int at = 0; at < BN / C::kAtom; ++at)
                      ptx::tma_load_2d(B_s + h * C::kBHalfBytes + at * C::kBAtomStride, &tmX,
                                       n0 + at * C::kAtom, run + h * 64, fb);
                  }
                }
              }
            }
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) {
            stop = true;
            break;
          }
        }
      }
    }
    if (lane == 0 && *abort_flag) {
      // wait (bounded) for the bulk / tensor copies of the last stages
      for (uint32_t k = (it > (uint32_t)C::kStages ? it - C::kStages : 0u); k < it; ++k) {
        ptx::mbar_wait(idx_bar(k % C::kStages), (k / C::kStages) & 1, a.status, nullptr);
        ptx::mbar_wait(full_bar(k % C::kStages), (k / C::kStages) & 1, a.status, nullptr);
        if constexpr (C::kSplitB)
          ptx::mbar_wait(full2_bar(k % C::kStages), (k / C::kStages) & 1, a.status, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_d = ptx::idesc_bf16(BN, 1, 0);
      const uint32_t idesc_s = ptx::idesc_bf16(BN, 1, 1);
      uint32_t it = 0, lu = 0;
      bool stop = false;
      for (int u = u_first; u < a.num_units && !stop; u += u_step, ++lu) {
        const int tile = u / a.nblk_n;
        const int4 info = tile_info_of(u, tile);
        const int nd = info.x, nblk = info.x + info.y;
        int kb0, kb1;
        k_range(nblk, kb0, kb1);
        const int b = (int)(lu % C::kAccBufs);
        if (!ptx::mbar_wait(acce_bar(b), ((lu / C::kAccBufs) & 1) ^ 1, a.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t acc = tmem + b * C::kAccCols;
        for (int kb = kb0; kb < kb1; ++kb, ++it) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1;
          const uint32_t accum0 = kb != kb0 ? 1u : 0u;  // first K-block overwrites
          if (!ptx::mbar_wait(full_bar(s), ph, a.status, abort_flag)) {
            stop = true;
            break;
          }
          ptx::fence_proxy_async_smem();  // cp.async (generic proxy) -> tensor-core reads
          ptx::tc_fence_after();
          const uint32_t A_s = ptx::smem_u32(smem + s * C::kStageBytes);
          const uint32_t B_s = A_s + C::kABytes;
          const uint32_t E_s = B_s + C::kBBytes;
          if (kb >= nd) {
            const uint32_t e_col = tmem + meta_col0 + 4 * s;
            // 128 lanes x 16 bytes, rows 16 B apart: core matrices of 8 rows, 128 B apart
            ptx::tc_cp_128x128b(e_col, ptx::smem_desc(E_s, 2048, 128, 0));
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              if (C::kSplitB && k == 2) {  // rows 64..127 of B
                if (!ptx::mbar_wait(full2_bar(s), ph, a.status, abort_flag)) {
                  stop = true;
                  break;
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_after();
              }
              const uint64_t ad = ptx::smem_desc(A_s + 32 * k, 16, 1024, 2);
              const uint64_t bd =
                  ptx::smem_desc(B_s + (k >> 1) * C::kBHalfBytes + 32 * (k & 1) * C::kAtomBytes,
                                 C::kBAtomStride, 8 * C::kAtomBytes, C::kBLayout);
              const uint32_t e = e_col + k;
              ptx::mma_sp_bf16(acc, ad, bd, e & ~1u, idesc_s | (e & 1u), (accum0 | k) ? 1u : 0u);
            }
            if (stop) break;
          } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint64_t ad = ptx::smem_desc(A_s + 32 * k, 16, 1024, 2);
              const uint64_t bd = ptx::smem_desc(B_s + 16 * k * C::kAtomBytes, C::kBAtomStride,
                                                 8 * C::kAtomBytes, C::kBLayout);
              ptx::mma_bf16(acc, ad, bd, idesc_d, (accum0 | k) ? 1u : 0u);
            }
            // a dense block has no second half: its barrier phase completes on the plain
            // arrivals; waiting keeps every phase consumed before the stage is reused
            if constexpr (C::kSplitB) {
              if (!ptx::mbar_wait(full2_bar(s), ph, a.status, abort_flag)) {
                stop = true;
                break;
              }
            }
          }
          ptx::tc_commit(empty_bar(s));
        }
        if (stop) break;
        ptx::tc_commit(accf_bar(b));  // accumulator b ready (immediately if no K-blocks)
      }
      // every tcgen05 operation issued above has completed once drain_bar flips
      ptx::tc_commit(drain_bar);
      ptx::mbar_wait(drain_bar, 0, a.status, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 5..8)
    const int q = warp & 3;  // tensor-memory lane quadrant this warp may access
    const int row = q * 32 + lane;
    constexpr int kChunk = BN >= 32 ? 32 : 16;
    uint32_t lu = 0;
    for (int u = u_first; u < a.num_units; u += u_step, ++lu) {
      const int tile = u / a.nblk_n, n0 = (u - tile * a.nblk_n) * BN;
      const int4 info = tile_info_of(u, tile);
      int kb0, kb1;
      k_range(info.x + info.y, kb0, kb1);
      const bool has = kb1 > kb0;  // else the accumulator was never written: zeros
      const int b = (int)(lu % C::kAccBufs);
      bool ok = ptx::mbar_wait(accf_bar(b), (lu / C::kAccBufs) & 1, a.status, abort_flag);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      if constexpr (SPLIT) {
        split_ready = true;
        split_has = has;
        split_tile = tile;
        split_n0 = n0;
        split_b = b;
        if (rank != 0) {
          // this CTA's partial -> the leader's reduction buffer, slot rank - 1
          const uint32_t dst = ptx::mapa_shared(ptx::smem_u32(red), 0) +
                               (uint32_t)((((rank - 1) * 128 + row) * BN) * 4);
          for (int col = 0; col < BN; col += kChunk) {
            uint32_t v[32];
            if (has) {
              const uint32_t taddr =
                  tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::kAccCols + col);
              if constexpr (kChunk == 32) ptx::tmem_ld_32x32b_x32(taddr, v);
              else ptx::tmem_ld_32x32b_x16(taddr, v);
              ptx::tmem_ld_wait();
            } else {
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = 0u;
            }
#pragma unroll
            for (int i = 0; i < kChunk; i += 4)
              ptx::st_cluster_v4(dst + (uint32_t)(col + i) * 4u, __uint_as_float(v[i]),
                                 __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                                 __uint_as_float(v[i + 3]));
          }
        }
      } else if constexpr (kChunk == 32) {
        // Per 32-column chunk: lane l holds row q*32 + l of the accumulator; it writes the
        // row into the warp's staging tile (16-byte pieces, slot = piece ^ (row & 7): no bank
        // conflict either way), and reads back piece l % 8 of row 4 i + l / 8, so that each
        // 16-byte store instruction writes 128 contiguous bytes of 4 rows of Y.
        const uint32_t ep = ptx::smem_u32(epi_stage + (warp & 3) * 4096);
        const bool epi = a.bias != nullptr || a.act != HINM_ACT_NONE;
        const float brow = (a.bias && row < a.T) ? __ldg(a.bias + tile * a.T + row) : 0.0f;
        for (int col = 0; col < BN; col += 32) {
          uint32_t v[32];
          if (has) {
            ptx::tmem_ld_32x32b_x32(
                tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::kAccCols + col), v);
            ptx::tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          if (epi) epi_apply<32>(v, brow, a.act);
          // columns of this chunk inside Y (a multiple of 8; <= 0 past N: nothing stored)
          const int cw = a.N - (n0 + col) < 32 ? a.N - (n0 + col) : 32;
          store_chunk32(a, ep, v, lane, q * 32, tile, n0 + col, cw);
        }
      } else {
        const bool row_ok = row < a.T;
        for (int col = 0; col < BN; col += kChunk) {
          uint32_t v[32];
          if (has) {
            const uint32_t taddr =
                tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(b * C::kAccCols + col);
            if constexpr (kChunk == 32) {
              ptx::tmem_ld_32x32b_x32(taddr, v);
            } else {
              ptx::tmem_ld_32x32b_x16(taddr, v);
            }
            ptx::tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          if (a.bias != nullptr || a.act != HINM_ACT_NONE)
            epi_apply<kChunk>(v, (a.bias && row_ok) ? __ldg(a.bias + tile * a.T + row) : 0.0f,
                              a.act);
          if (row_ok) store_row(a, v, kChunk, tile * a.T + row, n0 + col);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(acce_bar(b));  // accumulator b may be overwritten
    }
  }
  if constexpr (SPLIT) {
    // the partials of ranks 1.. are in the leader's shared memory after this barrier; the
    // leader adds them in rank order (deterministic) to its own and stores Y
    ptx::cluster_sync();
    if (rank == 0 && warp > C::kMmaWarp && split_ready) {
      ptx::tc_fence_after();
      const int q = warp & 3;
      const int row = q * 32 + lane;
      constexpr int kChunk = BN >= 32 ? 32 : 16;
      const bool row_ok = row < a.T;
      for (int col = 0; col < BN; col += kChunk) {
        uint32_t v[32];
        if (split_has) {
          const uint32_t taddr =
              tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(split_b * C::kAccCols + col);
          if constexpr (kChunk == 32) ptx::tmem_ld_32x32b_x32(taddr, v);
          else ptx::tmem_ld_32x32b_x16(taddr, v);
          ptx::tmem_ld_wait();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0u;
        }
        float o[32];
#pragma unroll
        for (int i = 0; i < kChunk; ++i) o[i] = __uint_as_float(v[i]);
        for (int r = 1; r < a.split; ++r) {
          const float* src = red + ((size_t)(r - 1) * 128 + row) * BN + col;
#pragma unroll
          for (int i = 0; i < kChunk; i += 4) {
            const float4 pv = *reinterpret_cast<const float4*>(src + i);
            o[i] = __fadd_rn(o[i], pv.x);
            o[i + 1] = __fadd_rn(o[i + 1], pv.y);
            o[i + 2] = __fadd_rn(o[i + 2], pv.z);
            o[i + 3] = __fadd_rn(o[i + 3], pv.w);
          }
        }
        uint32_t ob[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) ob[i] = i < kChunk ? __float_as_uint(o[i]) : 0u;
        if (a.bias != nullptr || a.act != HINM_ACT_NONE)
          epi_apply<kChunk>(ob, (a.bias && row_ok) ? __ldg(a.bias + split_tile * a.T + row) : 0.0f,
                            a.act);
        if (row_ok) store_row(a, ob, kChunk, split_tile * a.T + row, split_n0 + col);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ tile pairs
// Wide N with T = 128: work units are (tile pair 2p, 2p+1; 240-column block).  When the two
// tiles select the same X rows block by block (same block counts, and every block of both
// is the same ascending run: no vector pruned, or every vector dense), one B stage feeds the
// MMAs of both tiles, which halves the operand traffic that bounds the kernel.  Otherwise
// the unit runs the two tiles one after the other.  Tile q of the pair always accumulates in
// tensor-memory buffer q (2 x 240 columns + 16 metadata columns), so in a sequential unit the
// epilogue of one tile overlaps the main loop of the next.  The B stage is 4 column atoms of
// 64 (128-byte swizzle rows: full-width TMA rows, conflict-free gathers); a unit fills and
// multiplies its first 240 columns.
struct PairCfg {
  static constexpr int BN = 240;
  static constexpr int kAtom = 64;
  static constexpr int kAtoms = 4;
  static constexpr int kAtomBytes = 128;
  static constexpr int kSwzBits = 3;
  static constexpr int kChunksPerAtom = 8;
  static constexpr int kChunksPerRow = BN / 8;  // the gather fills 240 columns
  static constexpr int kBHalfBytes = 64 * kAtoms * kAtomBytes;
  static constexpr int kBBytes = 2 * kBHalfBytes;
  static constexpr int kBAtomStride = 64 * kAtomBytes;
  static constexpr int kEBytes = 2048;
  // stage: [A tile 0 | A tile 1 | B | E tile 0 | E tile 1]; a sequential unit uses the
  // tile-0 slots for either tile
  static constexpr int kAOff1 = kBlockBytes;
  static constexpr int kBOff = 2 * kBlockBytes;
  static constexpr int kEOff = kBOff + kBBytes;
  static constexpr int kStageBytes = kEOff + 2 * kEBytes;
  static constexpr int kIdxBytes = 512;
  static constexpr int kStages = 2;
  static constexpr uint32_t kBLayout = 2u;  // 128-byte swizzle
  static constexpr int kAccCols = BN;
  static constexpr int kMetaCol0 = 2 * BN;  // stage s, tile q: columns kMetaCol0 + 8 s + 4 q
  static constexpr int kTmemCols = 512;
  static constexpr int kEpiBytes = 4 * 32 * 32 * 4;
  static constexpr size_t kSmemBytes =
      (size_t)kStages * (kStageBytes + kIdxBytes) + 1024 /*align*/ + 512 /*barriers*/ + kEpiBytes;
  static constexpr bool kSplitB = true;
  static constexpr int kProducers = 128;
  static constexpr int kMmaWarp = 4;
  static constexpr int kBulkWarp = 9;
  static constexpr int kThreads = 320;
  static_assert(kStageBytes % 1024 == 0, "stage alignment");
  static_assert(kMetaCol0 + 8 * kStages <= kTmemCols, "tmem");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

// Warp-collective (every lane calls it with the same p): whether tiles 2p and 2p+1 read the
// same X rows block by block.  Gathered blocks (run -1) never count as shared.
__device__ __forceinline__ bool pair_shares_b(const SpmmArgs& a, int p, int lane) {
  const int t0 = 2 * p;
  if (t0 + 1 >= a.num_tiles) return false;
  const int4 i0 = __ldg(reinterpret_cast<const int4*>(a.tile_info) + t0);
  const int4 i1 = __ldg(reinterpret_cast<const int4*>(a.tile_info) + t0 + 1);
  if (i0.x != i1.x || i0.y != i1.y) return false;
  bool ok = true;
  for (int kb = lane; kb < i0.x + i0.y; kb += 32) {
    const bool sp = kb >= i0.x;
    const int r0 = sp ? __ldg(a.run_sparse + i0.w + kb - i0.x) : __ldg(a.run_dense + i0.z + kb);
    const int r1 = sp ? __ldg(a.run_sparse + i1.w + kb - i1.x) : __ldg(a.run_dense + i1.z + kb);
    ok = ok && r0 >= 0 && r0 == r1;
  }
  return __all_sync(0xffffffffu, ok);
}

// tmX3: X as (column, row, atom) with the atom stride 128 bytes inside a row, so that one
// box at column n0 covers columns n0 .. n0+255 of 64 rows (used while n0 + 256 <= N: every
// address stays in its row); tmX2: X as (column, row) with boxes of 64 x 64 (columns past N
// read as zeros), used for the last column block.
__global__ void __launch_bounds__(320, 1)
    spmm_pair_kernel(const __grid_constant__ CUtensorMap tmX3,
                     const __grid_constant__ CUtensorMap tmX2, const SpmmArgs a) {
  using C = PairCfg;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  ptx::enter_dependent();
  uint8_t* smem =
      reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* idx_region = smem + C::kStages * C::kStageBytes;  // [S][kIdxBytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(idx_region + C::kStages * C::kIdxBytes);
  // [0,S) full, [S,2S) empty, 2S+{0,1} accumulator full, 2S+{2,3} accumulator empty,
  // 2S+4 drain, [2S+5, 3S+5) index ready, [3S+5, 4S+5) second-half full; then the TMEM
  // address, the abort flag and one run flag per stage
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 4 * C::kStages + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* run_s = reinterpret_cast<volatile int*>(tmem_slot + 2);
  uint8_t* epi_stage = reinterpret_cast<uint8_t*>(bars) + 512;  // [4 warps][4 KB]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto full_bar = [&](int s) { return ptx::smem_u32(bars + s); };
  auto empty_bar = [&](int s) { return ptx::smem_u32(bars + C::kStages + s); };
  auto accf_bar = [&](int b) { return ptx::smem_u32(bars + 2 * C::kStages + b); };
  auto acce_bar = [&](int b) { return ptx::smem_u32(bars + 2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = ptx::smem_u32(bars + 2 * C::kStages + 4);
  auto idx_bar = [&](int s) { return ptx::smem_u32(bars + 2 * C::kStages + 5 + s); };
  auto full2_bar = [&](int s) { return ptx::smem_u32(bars + 3 * C::kStages + 5 + s); };
  auto info_of = [&](int t) { return __ldg(reinterpret_cast<const int4*>(a.tile_info) + t); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      ptx::mbar_init(full_bar(s), 1 + C::kProducers);
      ptx::mbar_init(empty_bar(s), 1);
      ptx::mbar_init(idx_bar(s), 1);
      ptx::mbar_init(full2_bar(s), 1 + C::kProducers);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(accf_bar(b), 1);
      ptx::mbar_init(acce_bar(b), 4);
    }
    ptx::mbar_init(drain_bar, 1);
    *abort_flag = 0;
    ptx::fence_mbar_init();
  }
  if (warp == C::kMmaWarp) {
    ptx::tmem_alloc(ptx::smem_u32(tmem_slot), C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int last_tile = a.num_tiles - 1;  // tile 2p + 1 exists iff 2p + 1 <= last_tile

  if (warp < 4) {
    // ------------------------------------------------------------ gather producers
    // As in spmm_kernel; every stop is warp-uniform (vote after each wait), because the
    // next unit starts with a warp-collective test.
    const int ptid = threadIdx.x;
    uint32_t it = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < a.num_units && !stop; u += gridDim.x) {
      const int p = u / a.nblk_n, n0 = (u - p * a.nblk_n) * BN;
      const bool pm = pair_shares_b(a, p, lane);
      const int nq = pm ? 1 : (2 * p + 1 <= last_tile ? 2 : 1);
      for (int q = 0; q < nq && !stop; ++q) {
        const int4 info = info_of(2 * p + q);
        const int nd = info.x, nblk = info.x + info.y;
        for (int kb = 0; kb < nblk; ++kb, ++it) {
          const bool sparse = kb >= nd;
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1;
          const bool ok = ptx::mbar_wait(idx_bar(s), ph, a.status, abort_flag);
          if (!__all_sync(0xffffffffu, ok)) {
            stop = true;
            break;
          }
          const int run = run_s[s];
          const uint32_t B_s = ptx::smem_u32(smem + s * C::kStageBytes + C::kBOff);
          const int* idx_s = reinterpret_cast<const int*>(idx_region + s * C::kIdxBytes);
          if (run < 0) {
            if (sparse) {
              using G = Gather<C, kSparseBK>;
              G gs;
              gs.load_index(idx_s, ptid);
              gs.template copy<0, G::kPer / 2>(B_s, a.X, a.N, n0, ptid);
              cp_async_arrive_noinc(full_bar(s));
              gs.template copy<G::kPer / 2, G::kPer>(B_s, a.X, a.N, n0, ptid);
              cp_async_arrive_noinc(full2_bar(s));
            } else {
              Gather<C, kDenseBK> gd;
              gd.load_index(idx_s, ptid);
              gd.copy(B_s, a.X, a.N, n0, ptid);
              cp_async_arrive_noinc(full_bar(s));
              ptx::mbar_arrive(full2_bar(s));
            }
          } else {
            ptx::mbar_arrive(full_bar(s));
            ptx::mbar_arrive(full2_bar(s));
          }
        }
      }
    }
    cp_async_wait_all();
  } else if (warp == C::kBulkWarp) {
    // ------------------------------------------------------------ bulk copies
    uint32_t it = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < a.num_units && !stop; u += gridDim.x) {
      const int p = u / a.nblk_n, n0 = (u - p * a.nblk_n) * BN;
      const bool pm = pair_shares_b(a, p, lane);
      if (lane == 0) {
        const int nq = pm ? 1 : (2 * p + 1 <= last_tile ? 2 : 1);
        for (int q = 0; q < nq && !stop; ++q) {
          const int4 info = info_of(2 * p + q);
          const int4 info1 = pm ? info_of(2 * p + 1) : info;
          const int nd = info.x, nblk = info.x + info.y;
          for (int kb = 0; kb < nblk; ++kb, ++it) {
            const bool sparse = kb >= nd;
            const size_t blk = sparse ? (size_t)(info.w + kb - nd) : (size_t)(info.z + kb);
            const size_t blk1 = sparse ? (size_t)(info1.w + kb - nd) : (size_t)(info1.z + kb);
            const int run = __ldg(sparse ? a.run_sparse + blk : a.run_dense + blk);
            const int s = it % C::kStages;
            const uint32_t ph = (it / C::kStages) & 1;
            if (!ptx::mbar_wait(empty_bar(s), ph ^ 1, a.status, abort_flag)) {
              stop = true;
              break;
            }
            const uint32_t A_s = ptx::smem_u32(smem + s * C::kStageBytes);
            const uint32_t B_s = A_s + C::kBOff;
            const uint32_t E_s = A_s + C::kEOff;
            const uint32_t I_s = ptx::smem_u32(idx_region + s * C::kIdxBytes);
            const int rows = sparse ? kSparseBK : kDenseBK;
            run_s[s] = run;  // published by the arrive below (release)
            if (run < 0) {
              ptx::mbar_arrive_expect_tx(idx_bar(s), (uint32_t)rows * 4u);
              ptx::bulk_g2s(I_s,
                            sparse ? a.idx_sparse + blk * kSparseBK : a.idx_dense + blk * kDenseBK,
                            (uint32_t)rows * 4u, idx_bar(s));
            } else {
              ptx::mbar_arrive(idx_bar(s));
            }
            // the full barrier takes A (both tiles' in a shared unit), the metadata and the
            // first 64 rows of a run; the second-half barrier the rest of the run
            const uint32_t na = pm ? 2u : 1u;
            const uint32_t bytes = na * (kBlockBytes + (sparse ? C::kEBytes : 0)) +
                                   (run >= 0 ? (uint32_t)C::kBHalfBytes : 0u);
            ptx::mbar_arrive_expect_tx(full_bar(s), bytes);
            ptx::mbar_arrive_expect_tx(full2_bar(s),
                                       run >= 0 && rows > 64 ? (uint32_t)C::kBHalfBytes : 0u);
            const uint16_t* vals = sparse ? a.vals_sparse : a.vals_dense;
            ptx::bulk_g2s(A_s, vals + blk * 8192, kBlockBytes, full_bar(s));
            if (pm) ptx::bulk_g2s(A_s + C::kAOff1, vals + blk1 * 8192, kBlockBytes, full_bar(s));
            if (sparse) {
              ptx::bulk_g2s(E_s, a.meta + blk * kMetaWords, C::kEBytes, full_bar(s));
              if (pm)
                ptx::bulk_g2s(E_s + C::kEBytes, a.meta + blk1 * kMetaWords, C::kEBytes,
                              full_bar(s));
            }
            if (run >= 0) {
#pragma unroll 1
              for (int h = 0; h < rows / 64; ++h) {
                const uint32_t fb = h == 1 ? full2_bar(s) : full_bar(s);
                if (a.x3d && n0 + C::kAtoms * C::kAtom <= a.N) {
                  ptx::tma_load_3d(B_s + h * C::kBHalfBytes, &tmX3, n0, run + h * 64, 0, fb);
                } else {
#pragma unroll 1
                  for (int at = 0; at < C::kAtoms; ++at)
                    ptx::tma_load_2d(B_s + h * C::kBHalfBytes + at * C::kBAtomStride, &tmX2,
                                     n0 + at * C::kAtom, run + h * 64, fb);
                }
              }
            }
          }
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
    }
    if (lane == 0 && *abort_flag) {
      // wait (bounded) for the bulk / tensor copies of the last stages
      for (uint32_t k = (it > (uint32_t)C::kStages ? it - C::kStages : 0u); k < it; ++k) {
        ptx::mbar_wait(idx_bar(k % C::kStages), (k / C::kStages) & 1, a.status, nullptr);
        ptx::mbar_wait(full_bar(k % C::kStages), (k / C::kStages) & 1, a.status, nullptr);
        ptx::mbar_wait(full2_bar(k % C::kStages), (k / C::kStages) & 1, a.status, nullptr);
      }
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    uint32_t it = 0, lu0 = 0, lu1 = 0;
    bool stop = false;
    for (int u = blockIdx.x; u < a.num_units && !stop; u += gridDim.x) {
      const int p = u / a.nblk_n, n0 = (u - p * a.nblk_n) * BN;
      const bool pm = pair_shares_b(a, p, lane);
      if (lane == 0) {
        const int w = a.N - n0 < BN ? a.N - n0 : BN;
        const int nmma = (w + 15) & ~15;  // MMA width: the unit's columns, rounded up to 16
        const uint32_t idesc_d = ptx::idesc_bf16(nmma, 1, 0);
        const uint32_t idesc_s = ptx::idesc_bf16(nmma, 1, 1);
        const int nq = pm ? 1 : (2 * p + 1 <= last_tile ? 2 : 1);
        for (int q = 0; q < nq && !stop; ++q) {
          // buffers this pass writes: both in a shared unit, else buffer q
          if (pm || q == 0) {
            if (!ptx::mbar_wait(acce_bar(0), (lu0 & 1) ^ 1, a.status, abort_flag)) {
              stop = true;
              break;
            }
          }
          if (pm || q == 1) {
            if (!ptx::mbar_wait(acce_bar(1), (lu1 & 1) ^ 1, a.status, abort_flag)) {
              stop = true;
              break;
            }
          }
          ptx::tc_fence_after();
          const uint32_t acc0 = tmem + (uint32_t)(q * C::kAccCols);  // this pass's tile
          const uint32_t acc1 = tmem + (uint32_t)C::kAccCols;        // tile 1 of a shared unit
          const int4 info = info_of(2 * p + q);
          const int nd = info.x, nblk = info.x + info.y;
          for (int kb = 0; kb < nblk; ++kb, ++it) {
            const int s = it % C::kStages;
            const uint32_t ph = (it / C::kStages) & 1;
            const uint32_t accum0 = kb != 0 ? 1u : 0u;  // first K-block overwrites
            if (!ptx::mbar_wait(full_bar(s), ph, a.status, abort_flag)) {
              stop = true;
              break;
            }
            ptx::fence_proxy_async_smem();  // cp.async (generic proxy) -> tensor-core reads
            ptx::tc_fence_after();
            const uint32_t A_s = ptx::smem_u32(smem + s * C::kStageBytes);
            const uint32_t B_s = A_s + C::kBOff;
            const uint32_t E_s = A_s + C::kEOff;
            if (kb >= nd) {
              const uint32_t e0 = tmem + (uint32_t)(C::kMetaCol0 + 8 * s);
              const uint32_t e1 = e0 + 4;
              ptx::tc_cp_128x128b(e0, ptx::smem_desc(E_s, 2048, 128, 0));
              if (pm) ptx::tc_cp_128x128b(e1, ptx::smem_desc(E_s + C::kEBytes, 2048, 128, 0));
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                if (k == 2) {  // rows 64..127 of B
                  if (!ptx::mbar_wait(full2_bar(s), ph, a.status, abort_flag)) {
                    stop = true;
                    break;
                  }
                  ptx::fence_proxy_async_smem();
                  ptx::tc_fence_after();
                }
                const uint64_t bd =
                    ptx::smem_desc(B_s + (k >> 1) * C::kBHalfBytes + 32 * (k & 1) * C::kAtomBytes,
                                   C::kBAtomStride, 8 * C::kAtomBytes, C::kBLayout);
                const uint32_t acc_on = (accum0 | k) ? 1u : 0u;
                const uint32_t f0 = e0 + k;
                ptx::mma_sp_bf16(acc0, ptx::smem_desc(A_s + 32 * k, 16, 1024, 2), bd, f0 & ~1u,
                                 idesc_s | (f0 & 1u), acc_on);
                if (pm) {
                  const uint32_t f1 = e1 + k;
                  ptx::mma_sp_bf16(acc1, ptx::smem_desc(A_s + C::kAOff1 + 32 * k, 16, 1024, 2),
                                   bd, f1 & ~1u, idesc_s | (f1 & 1u), acc_on);
                }
              }
              if (stop) break;
            } else {
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint64_t bd = ptx::smem_desc(B_s + 16 * k * C::kAtomBytes, C::kBAtomStride,
                                                   8 * C::kAtomBytes, C::kBLayout);
                const uint32_t acc_on = (accum0 | k) ? 1u : 0u;
                ptx::mma_bf16(acc0, ptx::smem_desc(A_s + 32 * k, 16, 1024, 2), bd, idesc_d,
                              acc_on);
                if (pm)
                  ptx::mma_bf16(acc1, ptx::smem_desc(A_s + C::kAOff1 + 32 * k, 16, 1024, 2), bd,
                                idesc_d, acc_on);
              }
              // a dense block has no second half: its barrier phase completes on the plain
              // arrivals; waiting keeps every phase consumed before the stage is reused
              if (!ptx::mbar_wait(full2_bar(s), ph, a.status, abort_flag)) {
                stop = true;
                break;
              }
            }
            ptx::tc_commit(empty_bar(s));
          }
          if (stop) break;
          // accumulator(s) ready (immediately if the tile has no K-blocks)
          if (pm || q == 0) {
            ptx::tc_commit(accf_bar(0));
            ++lu0;
          }
          if (pm || q == 1) {
            ptx::tc_commit(accf_bar(1));
            ++lu1;
          }
        }
      }
      stop = __shfl_sync(0xffffffffu, stop ? 1 : 0, 0) != 0;
    }
    if (lane == 0) {
      // every tcgen05 operation issued above has completed once drain_bar flips
      ptx::tc_commit(drain_bar);
      ptx::mbar_wait(drain_bar, 0, a.status, nullptr);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 5..8)
    // Tile q of each unit from buffer q; per 32-column chunk the lanes' accumulator rows go
    // through the warp's swizzled shared tile and out as 128-byte row segments of Y.
    const int qd = warp & 3;  // tensor-memory lane quadrant this warp may access
    const uint32_t ep = ptx::smem_u32(epi_stage + qd * 4096);
    const bool epi = a.bias != nullptr || a.act != HINM_ACT_NONE;
    uint32_t lu[2] = {0u, 0u};
    bool stop = false;
    for (int u = blockIdx.x; u < a.num_units && !stop; u += gridDim.x) {
      const int p = u / a.nblk_n, n0 = (u - p * a.nblk_n) * BN;
      const int w = a.N - n0 < BN ? a.N - n0 : BN;
      const int nq = 2 * p + 1 <= last_tile ? 2 : 1;
      for (int q = 0; q < nq; ++q) {
        const int tile = 2 * p + q;
        const int4 info = info_of(tile);
        const bool has = info.x + info.y > 0;  // else the accumulator was never written
        const bool ok = ptx::mbar_wait(accf_bar(q), lu[q] & 1, a.status, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) {
          stop = true;
          break;
        }
        ++lu[q];
        ptx::tc_fence_after();
        const float brow = a.bias ? __ldg(a.bias + tile * a.T + qd * 32 + lane) : 0.0f;
        for (int col = 0; col < w; col += 32) {
          const int cw = w - col < 32 ? w - col : 32;  // a multiple of 8
          uint32_t v[32];
          if (has) {
            const uint32_t taddr =
                tmem + ((uint32_t)(qd * 32) << 16) + (uint32_t)(q * C::kAccCols + col);
            if (cw > 16) ptx::tmem_ld_32x32b_x32(taddr, v);
            else ptx::tmem_ld_32x32b_x16(taddr, v);
            ptx::tmem_ld_wait();
          } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
          }
          if (epi) epi_apply<32>(v, brow, a.act);
          store_chunk32(a, ep, v, lane, qd * 32, tile, n0 + col, cw);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(acce_bar(q));  // buffer q may be overwritten
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ------------------------------------------------------------------ host side
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// X (K rows x N bf16, row-major) as a 2-D tensor map swizzled like the B operand (atom * 2
// bytes per swizzle row), box 64 rows x `atom` columns; columns past N read as zeros.
bool make_x_map_2d(CUtensorMap* m, const uint16_t* X, int K, int N, int atom) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)K};
  cuuint64_t strides[1] = {(cuuint64_t)N * 2};
  cuuint32_t box[2] = {(cuuint32_t)atom, (cuuint32_t)(K < 64 ? K : 64)};
  cuuint32_t estr[2] = {1, 1};
  const CUtensorMapSwizzle sw = atom == 64   ? CU_TENSOR_MAP_SWIZZLE_128B
                                : atom == 32 ? CU_TENSOR_MAP_SWIZZLE_64B
                                             : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(X), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// The tensor map of spmm_kernel.  With 64-column atoms and N a multiple of 64 it is 3-D
// (column within the atom, row, atom; the atom stride is 128 bytes) with a box of all the
// unit's atoms for 64 rows, so one load fills a half of the B tile; else the 2-D map.
bool make_x_map(CUtensorMap* m, const uint16_t* X, int K, int N, int atom, int atoms, bool* x3d) {
  auto fn = encode_fn();
  if (!fn) return false;
  *x3d = false;
  if (atom == 64 && N % 64 == 0 && K >= 64 && atoms <= 4) {
    cuuint64_t dims[3] = {64, (cuuint64_t)K, (cuuint64_t)(N / 64)};
    cuuint64_t strides[2] = {(cuuint64_t)N * 2, 128};
    cuuint32_t box[3] = {64, 64, (cuuint32_t)atoms};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(X), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r == CUDA_SUCCESS) {
      *x3d = true;
      return true;
    }
  }
  return make_x_map_2d(m, X, K, N, atom);
}

// X as (column, row, atom): dims {N, K, atoms}, the atom stride `atom` columns within the
// row, so that a box of {atom, 64, atoms} at column n0 reads columns n0 .. n0 + atom*atoms - 1
// of 64 rows.  Columns are bounds-checked only against N along the first dimension: the
// caller uses it only for boxes with n0 + atom*atoms <= N.  false if the driver refuses it.
bool make_x_row_atoms_map(CUtensorMap* m, const uint16_t* X, int K, int N, int atom, int atoms) {
  auto fn = encode_fn();
  if (!fn || K < 64 || N < atom * atoms) return false;
  cuuint64_t dims[3] = {(cuuint64_t)N, (cuuint64_t)K, (cuuint64_t)atoms};
  cuuint64_t strides[2] = {(cuuint64_t)N * 2, (cuuint64_t)atom * 2};
  cuuint32_t box[3] = {(cuuint32_t)atom, 64, (cuuint32_t)atoms};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(X), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

template <int BN, bool SPLIT>
cudaError_t run(const hinm_layout& L, const uint16_t* X, int N, const SpmmOut& o, int split, int* status,
                cudaStream_t s) {
  using C = SpmmCfg<BN, SPLIT>;
  cudaError_t attr_err =
      set_max_dynamic_smem((const void*)spmm_kernel<BN, SPLIT>, (int)C::kSmemBytes);
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap map;
  bool x3d = false;
  if (!make_x_map(&map, X, L.K, N, C::kAtom, BN / C::kAtom, &x3d)) return cudaErrorInvalidValue;
  const int nblk_n = (N + BN - 1) / BN;
  const int units = L.num_tiles * nblk_n;
  SpmmArgs a{L.tile_info, L.vals_dense, L.vals_sparse, L.meta,   L.idx_dense, L.idx_sparse,
             L.run_dense, L.run_sparse, X,             o.Y,      N,           L.T,
             L.num_tiles, nblk_n,       units,         SPLIT ? split : 1,       x3d ? 1 : 0,
             status,      o.bias,       o.act,         o.Yb};
  if constexpr (!SPLIT) {
    const int grid = units < num_sms() ? units : num_sms();
    return launch_kernel(spmm_kernel<BN, false>, grid, C::kThreads, C::kSmemBytes, s, nullptr,
                         map, a);
  } else {
    // one cluster of `split` CTAs per unit
    cudaLaunchAttribute cluster;
    cluster.id = cudaLaunchAttributeClusterDimension;
    cluster.val.clusterDim.x = (unsigned)split;
    cluster.val.clusterDim.y = 1;
    cluster.val.clusterDim.z = 1;
    return launch_kernel(spmm_kernel<BN, true>, (unsigned)(units * split), C::kThreads,
                         C::kSmemBytes, s, &cluster, map, a);
  }
}

// Tile pairs x 240-column blocks (T = 128, wide N).
constexpr int kPairMinN = 1024;
cudaError_t run_pair(const hinm_layout& L, const uint16_t* X, int N, const SpmmOut& o, int* status,
                     cudaStream_t s) {
  using C = PairCfg;
  cudaError_t attr_err = set_max_dynamic_smem((const void*)spmm_pair_kernel, (int)C::kSmemBytes);
  if (attr_err != cudaSuccess) return attr_err;
  CUtensorMap map3, map2;
  if (!make_x_map_2d(&map2, X, L.K, N, C::kAtom)) return cudaErrorInvalidValue;
  const bool x3d = make_x_row_atoms_map(&map3, X, L.K, N, C::kAtom, C::kAtoms);
  if (!x3d) map3 = map2;
  const int nblk_n = (N + C::BN - 1) / C::BN;
  const int units = (L.num_tiles + 1) / 2 * nblk_n;
  SpmmArgs a{L.tile_info, L.vals_dense, L.vals_sparse, L.meta,   L.idx_dense, L.idx_sparse,
             L.run_dense, L.run_sparse, X,             o.Y,      N,           L.T,
             L.num_tiles, nblk_n,       units,         1,        x3d ? 1 : 0, status,
             o.bias,      o.act,        o.Yb};
  const int grid = units < num_sms() ? units : num_sms();
  return launch_kernel(spmm_pair_kernel, grid, C::kThreads, C::kSmemBytes, s, nullptr, map3, map2,
                       a);
}

// Split-K when the units (tile x column block) fill less than half of the SMs: each unit's
// K-blocks are shared by a cluster of up to kMaxSplit CTAs.
template <int BN>
cudaError_t run_auto(const hinm_layout& L, const uint16_t* X, int N, const SpmmOut& o, int* status,
                     cudaStream_t s) {
  const int units = L.num_tiles * ((N + BN - 1) / BN);
  if constexpr (BN <= 32) {
    int split = units > 0 ? num_sms() / units : 1;
    if (split > SpmmCfg<BN, true>::kMaxSplit) split = SpmmCfg<BN, true>::kMaxSplit;
    if (split >= 2) return run<BN, true>(L, X, N, o, split, status, s);
  }
  return run<BN, false>(L, X, N, o, 1, status, s);
}

}  // namespace

cudaError_t launch_spmm(const hinm_layout& L, const uint16_t* X, int N, const SpmmOut& o,
                        bool tile_pairs, int* status, cudaStream_t s) {
  if (N <= 16) return run_auto<16>(L, X, N, o, status, s);
  if (N <= 32) return run_auto<32>(L, X, N, o, status, s);
  if (N <= 64) return run_auto<64>(L, X, N, o, status, s);
  if (N < 256) return run_auto<128>(L, X, N, o, status, s);
  if (tile_pairs && L.T == 128 && N >= kPairMinN) return run_pair(L, X, N, o, status, s);
  // 192 columns per unit at wide N: a 66 KB stage leaves room for three stages (256 columns
  // fit two), and the third stage's copies in flight outweigh reading the A blocks once per
  // 192 instead of 256 columns (measured on B200: HiNM up-proj 198.7 -> 172.0 us, gate
  // 11008x4096x512 64.3 -> 47.1 us, Y bit for bit the same)
  return run_auto<192>(L, X, N, o, status, s);
}

}  // namespace hinm
