// a1. Importance: s_c = sum_n x_cn^2 (fp64, n ascending, rounded once to fp32) and
// I[i,c] = fl32(fl32(w_ic^2) * s_c)  (FlexHiNM-GP notes, 关键设计 1/2: second-order
// importance, importance matrix D; diagonal proxy w^2 ||x_c||^2).
//
// Both kernels are HBM streams.  channel_energy reads X once (one warp per channel,
// 16-byte loads along its row); importance reads W once and writes I once, 4 elements
// per thread with 8-byte loads and 16-byte stores, grid-stride over the matrix.
#include <cuda_bf16.h>

#include <mutex>

#include "hinm_internal.h"
#include "launch.cuh"
#include "ptx.cuh"

namespace hinm {
namespace {

__device__ __forceinline__ double bf16_to_f64(uint32_t bits16) {
  return static_cast<double>(__uint_as_float(bits16 << 16));
}

// One warp per channel.  s_c is fl32 of the sequential fp64 sum of x_cn^2 over n ascending.
// The warp adds the squares in its own order instead (per lane, then a shuffle tree).  The
// squares of bf16 values are exact in fp64, and for N non-negative terms every order of fp64
// additions, the sequential one included, ends within gamma = (N-1) 2^-53 / (1 - (N-1) 2^-53)
// (relative) of the exact sum; so the sequential result lies in [p (1 - d), p (1 + d)] with
// d = 4 N 2^-53 > 2.01 gamma, p the warp's sum.  When both ends of that interval round to the
// same fp32 value, that value is fl32 of the sequential sum (rounding is monotone).  Otherwise
// (p within about N 2^-51 of an fp32 rounding boundary, or not finite: rare) lane 0 runs the
// sequential chain itself.
constexpr int kEnergyWarps = 8;

// zero_int (nullptr allowed): n_zero ints of a later kernel cleared by the grid on the way
// (the tile maxima that importance_stats_kernel raises with atomicMax)
__global__ void __launch_bounds__(kEnergyWarps * 32) channel_energy_kernel(
    const uint16_t* __restrict__ X, int K, int N, float* __restrict__ s,
    int* __restrict__ zero_int, int n_zero) {
  ptx::enter_dependent();
  if (zero_int)
    for (int x = blockIdx.x * blockDim.x + threadIdx.x; x < n_zero; x += gridDim.x * blockDim.x)
      zero_int[x] = 0;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x * kEnergyWarps + (threadIdx.x >> 5);
  if (c >= K) return;  // warp-uniform
  const uint16_t* row = X + (size_t)c * N;
  double p = 0.0;
#pragma unroll 4
  for (int base = lane * 8; base < N; base += 32 * 8) {  // N % 8 == 0: whole 16-byte pieces
    const uint4 q = __ldg(reinterpret_cast<const uint4*>(row + base));
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const double a = bf16_to_f64(w[h] & 0xFFFFu);
      const double b = bf16_to_f64(w[h] >> 16);
      p = __dadd_rn(p, __dadd_rn(__dmul_rn(a, a), __dmul_rn(b, b)));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) p = __dadd_rn(p, __shfl_xor_sync(0xffffffffu, p, o));
  if (lane == 0) {
    const double d = __dmul_rn(p, __dmul_rn((double)N, 0x1p-51));
    const float lo = __double2float_rn(__dsub_rn(p, d));
    const float hi = __double2float_rn(__dadd_rn(p, d));
    float r = lo;
    if (!(lo == hi)) {
      double acc = 0.0;  // the sequential chain, n ascending
      for (int n = 0; n < N; ++n) {
        const double v = bf16_to_f64(row[n]);
        acc = __dadd_rn(acc, __dmul_rn(v, v));
      }
      r = __double2float_rn(acc);
    }
    s[c] = r;
  }
}

// 4 consecutive elements of one row per quad (K % 4 == 0); each thread takes kQuads quads
// per pass of the grid-stride loop, their loads issued before any arithmetic.
constexpr int kQuads = 4;

__global__ void importance_kernel(const uint16_t* __restrict__ W, const float* __restrict__ s,
                                  int M, int K, float* __restrict__ I) {
  ptx::enter_dependent();
  const long long total4 = (long long)M * K / 4;
  const int k4 = K / 4;
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long q0 = blockIdx.x * (long long)blockDim.x + threadIdx.x; q0 < total4;
       q0 += stride * kQuads) {
    uint2 wv[kQuads];
    float4 sv[kQuads];
#pragma unroll
    for (int u = 0; u < kQuads; ++u) {
      const long long q = q0 + u * stride;
      if (q < total4) {
        wv[u] = __ldg(reinterpret_cast<const uint2*>(W) + q);
        sv[u] = __ldg(reinterpret_cast<const float4*>(s + (int)(q % k4) * 4));
      }
    }
#pragma unroll
    for (int u = 0; u < kQuads; ++u) {
      const long long q = q0 + u * stride;
      if (q >= total4) break;
      const float w0 = __uint_as_float(wv[u].x << 16), w1 = __uint_as_float(wv[u].x & 0xFFFF0000u);
      const float w2 = __uint_as_float(wv[u].y << 16), w3 = __uint_as_float(wv[u].y & 0xFFFF0000u);
      float4 o;
      o.x = __fmul_rn(__fmul_rn(w0, w0), sv[u].x);
      o.y = __fmul_rn(__fmul_rn(w1, w1), sv[u].y);
      o.z = __fmul_rn(__fmul_rn(w2, w2), sv[u].z);
      o.w = __fmul_rn(__fmul_rn(w3, w3), sv[u].w);
      __stcs(reinterpret_cast<float4*>(I) + q, o);
    }
  }
}

// I as importance_kernel computes it, and with it the boundary search's tile statistics:
// V[t, c] = the fp64 sum of the tile's I[., c] over its rows in ascending order (the same
// additions in the same order as the search's own vector scores), and tile_pmax[t] = the
// exponent index p (value = m 2^(p-149)) of the tile's largest importance.  A CTA of 256
// threads takes 512 channels of one tile; the tile's rows of W for them come into shared
// memory 32 at a time by cp.async (two buffers: the next 32 rows land while these are
// summed), and each thread walks its 2 channels down the rows in ascending order.
// tile_pmax must be 0 before the launch.
constexpr int kStatRows = 32;      // rows per buffer; T is a multiple of 32 (64 or 128)
constexpr int kStatThreads = 256;  // 2 channels each: 512 channels (1 KB of a row) per CTA
constexpr int kStatChans = 2 * kStatThreads;
constexpr size_t kStatBufBytes = (size_t)kStatRows * kStatChans * sizeof(uint16_t);  // 32 KB

__global__ void __launch_bounds__(kStatThreads) importance_stats_kernel(
    const uint16_t* __restrict__ W, const float* __restrict__ s, int K, int T,
    float* __restrict__ I, double* __restrict__ V, int* __restrict__ tile_pmax) {
  extern __shared__ __align__(16) uint8_t stat_smem[];  // [2][kStatRows][kStatChans] bf16
  ptx::enter_dependent();
  const int c_base = blockIdx.x * kStatChans;
  const int t = blockIdx.y;
  const int nch = min(kStatChans, K - c_base);  // channels of this CTA (a multiple of 4)
  const uint16_t* wt = W + (size_t)t * T * K + c_base;
  const uint32_t buf0 = ptx::smem_u32(stat_smem);
  auto issue = [&](int r0, int b) {  // rows r0 .. r0 + 31 of the tile -> buffer b
    const uint32_t dst = buf0 + (uint32_t)(b * kStatBufBytes);
    if ((K & 7) == 0) {  // 16-byte pieces (8 channels), never straddling K
      const int per_row = nch >> 3;
      for (int q = threadIdx.x; q < kStatRows * per_row; q += kStatThreads) {
        const int r = q / per_row, x = q - r * per_row;
        ptx::cp_async16(dst + (uint32_t)(r * kStatChans * 2 + 16 * x),
                        wt + (size_t)(r0 + r) * K + 8 * x);
      }
    } else {  // 8-byte pieces (4 channels)
      const int per_row = nch >> 2;
      for (int q = threadIdx.x; q < kStatRows * per_row; q += kStatThreads) {
        const int r = q / per_row, x = q - r * per_row;
        ptx::cp_async8(dst + (uint32_t)(r * kStatChans * 2 + 8 * x),
                       wt + (size_t)(r0 + r) * K + 4 * x);
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  issue(0, 0);
  if (kStatRows < T) issue(kStatRows, 1);

  const int c0 = 2 * threadIdx.x;  // this thread's channel pair within the CTA
  const bool mine = c0 < nch;
  const float s0 = mine ? __ldg(s + c_base + c0) : 0.0f, s1 = mine ? __ldg(s + c_base + c0 + 1) : 0.0f;
  float2* ip = (I && mine) ? reinterpret_cast<float2*>(I + (size_t)t * T * K + c_base + c0) : nullptr;
  const size_t step = (size_t)K / 2;  // one row, in channel pairs
  double v0 = 0.0, v1 = 0.0;
  uint32_t mb = 0;  // largest bit pattern = largest value (non-negative floats)
  for (int r0 = 0, b = 0; r0 < T; r0 += kStatRows, b ^= 1) {
    // this buffer's copies have landed when at most the next buffer's group is pending
    if (r0 + kStatRows < T) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    if (mine) {
      const uint32_t* rows = reinterpret_cast<const uint32_t*>(stat_smem + b * kStatBufBytes) + threadIdx.x;
#pragma unroll 8
      for (int k = 0; k < kStatRows; ++k) {  // rows ascending
        const uint32_t wv = rows[k * kStatThreads];
        const float w0 = __uint_as_float(wv << 16), w1 = __uint_as_float(wv & 0xFFFF0000u);
        const float i0 = __fmul_rn(__fmul_rn(w0, w0), s0);
        const float i1 = __fmul_rn(__fmul_rn(w1, w1), s1);
        if (ip) __stcs(ip + (size_t)(r0 + k) * step, make_float2(i0, i1));
        v0 = __dadd_rn(v0, (double)i0);
        v1 = __dadd_rn(v1, (double)i1);
        mb = max(mb, max(__float_as_uint(i0), __float_as_uint(i1)));
      }
    }
    __syncthreads();  // buffer b is refilled next
    if (r0 + 2 * kStatRows < T) issue(r0 + 2 * kStatRows, b);
  }
  if (mine) {
    V[(size_t)t * K + c_base + c0] = v0;
    V[(size_t)t * K + c_base + c0 + 1] = v1;
  }
  int pm = 0;
  if (mb) {
    const uint32_t e = mb >> 23;
    pm = (e ? (int)e : 1) - 1;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) pm = max(pm, __shfl_xor_sync(0xffffffffu, pm, o));
  if ((threadIdx.x & 31) == 0) atomicMax(tile_pmax + t, pm);
}

int sm_count() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

// Scratch of the workspace-free entry point: the channel energies s_c of one call.  One copy
// per device; nothing in it has to start at zero (channel_energy_kernel writes s_c for every
// c < K before importance_kernel reads it, in stream order).
static __device__ __align__(256) float g_noalloc_energy[kNoAllocMaxK];

SymbolCache g_noalloc_cache;

}  // namespace

// Address of the static scratch on the current device (the caller's current device is the
// one the call runs on), resolved with cudaGetSymbolAddress once per device and context.
cudaError_t noalloc_energy_scratch(float** out) {
  void* p = nullptr;
  cudaError_t e = resolve_symbol(g_noalloc_cache, &g_noalloc_energy, &p);
  *out = static_cast<float*>(p);
  return e;
}

size_t tile_stats_v_bytes(int M, int K, int T) {
  return ((size_t)(M / T) * K * sizeof(double) + 255) & ~size_t(255);
}
size_t tile_stats_s_offset(int M, int K, int T) {
  return tile_stats_v_bytes(M, K, T) + (((size_t)(M / T) * sizeof(int) + 255) & ~size_t(255));
}
size_t tile_stats_bytes(int M, int K, int T) {
  return tile_stats_s_offset(M, K, T) + (((size_t)K * sizeof(float) + 255) & ~size_t(255));
}

cudaError_t launch_importance_stats(const uint16_t* W, const uint16_t* X, int M, int K, int N,
                                    int T, float* I, void* stats, cudaStream_t st) {
  // the channel energies live in the statistics, so that I can be recomputed from W later
  float* s_scratch = reinterpret_cast<float*>(static_cast<char*>(stats) +
                                              tile_stats_s_offset(M, K, T));
  const int nt = M / T;
  double* V = static_cast<double*>(stats);
  int* pmax = reinterpret_cast<int*>(static_cast<char*>(stats) + tile_stats_v_bytes(M, K, T));
  // the energies' grid also clears the tile maxima (raised by importance_stats_kernel next)
  const unsigned ge = (K + kEnergyWarps - 1) / kEnergyWarps;
  cudaError_t e = launch_kernel(channel_energy_kernel, ge, kEnergyWarps * 32, 0, st, nullptr, X,
                                K, N, s_scratch, pmax, nt);
  if (e != cudaSuccess) return e;
  const size_t smem = 2 * kStatBufBytes;
  e = set_max_dynamic_smem((const void*)importance_stats_kernel, (int)smem);
  if (e != cudaSuccess) return e;
  const dim3 g((K + kStatChans - 1) / kStatChans, nt);
  return launch_kernel(importance_stats_kernel, g, kStatThreads, smem, st, nullptr, W, s_scratch,
                       K, T, I, V, pmax);
}

size_t importance_workspace_bytes(int K) { return ((size_t)K * sizeof(float) + 255) & ~size_t(255); }

cudaError_t launch_importance(const uint16_t* W, const uint16_t* X, int M, int K, int N,
                              float* I, float* s_scratch, cudaStream_t st) {
  const unsigned ge = (K + kEnergyWarps - 1) / kEnergyWarps;
  cudaError_t e = launch_kernel(channel_energy_kernel, ge, kEnergyWarps * 32, 0, st, nullptr, X,
                                K, N, s_scratch, nullptr, 0);
  if (e != cudaSuccess) return e;
  const long long total4 = (long long)M * K / 4;
  long long blocks = (total4 + 255) / 256;
  const long long cap = (long long)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  return launch_kernel(importance_kernel, (unsigned)blocks, 256, 0, st, nullptr, W, s_scratch, M,
                       K, I);
}

}  // namespace hinm
