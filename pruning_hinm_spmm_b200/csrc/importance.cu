// a1. Importance: s_c = sum_n x_cn^2 (fp64, n ascending, rounded once to fp32) and
// I[i,c] = fl32(fl32(w_ic^2) * s_c)  (FlexHiNM-GP notes, 关键设计 1/2: second-order
// importance, importance matrix D; diagonal proxy w^2 ||x_c||^2).
//
// Both kernels are HBM streams.  channel_energy reads X once (one thread per channel,
// 16-byte loads along its row); importance reads W once and writes I once, 4 elements
// per thread with 8-byte loads and 16-byte stores, grid-stride over the matrix.
#include <cuda_bf16.h>

#include <mutex>

#include "hinm_internal.h"

namespace hinm {
namespace {

__device__ __forceinline__ double bf16_to_f64(uint32_t bits16) {
  return static_cast<double>(__uint_as_float(bits16 << 16));
}

// One CTA per 32 channels.  The order of the sum is fixed (n ascending, one fp64 chain per
// channel), so the sum itself cannot be split; what is parallel is the loading.  All 128
// threads stage [32 channels x 256 values] chunks of X into shared memory with 16-byte
// cp.async, double-buffered, while warp 0 runs the 32 chains over the previous chunk
// (lane = channel; rows padded by 16 bytes so the 16-byte reads are conflict-free).
constexpr int kEnergyChannels = 32;
constexpr int kEnergyChunk = 256;                      // values per channel per chunk
constexpr int kEnergyRowBytes = kEnergyChunk * 2 + 16;  // padded row
constexpr int kEnergyThreads = 128;

__device__ __forceinline__ void energy_cp16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

__global__ void __launch_bounds__(kEnergyThreads) channel_energy_kernel(
    const uint16_t* __restrict__ X, int K, int N, float* __restrict__ s) {
  __shared__ __align__(16) uint8_t buf[2][kEnergyChannels * kEnergyRowBytes];
  const int c0 = blockIdx.x * kEnergyChannels;
  const int nch = min(kEnergyChannels, K - c0);
  const int nchunks = (N + kEnergyChunk - 1) / kEnergyChunk;
  constexpr int kPieces = kEnergyChunk / 8;  // 16-byte pieces per channel per chunk

  auto stage = [&](int chunk, int b) {
    const int n0 = chunk * kEnergyChunk;
    const int pieces = min(kPieces, (N - n0) / 8);
    const uint32_t base = (uint32_t)__cvta_generic_to_shared(buf[b]);
    for (int q = threadIdx.x; q < kEnergyChannels * kPieces; q += kEnergyThreads) {
      const int ch = q / kPieces, p = q - ch * kPieces;
      if (ch < nch && p < pieces)
        energy_cp16(base + ch * kEnergyRowBytes + p * 16, X + (size_t)(c0 + ch) * N + n0 + p * 8);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };

  double acc = 0.0;
  stage(0, 0);
  for (int chunk = 0; chunk < nchunks; ++chunk) {
    if (chunk + 1 < nchunks) {
      stage(chunk + 1, (chunk + 1) & 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x < nch) {
      const int nv = min(kEnergyChunk, N - chunk * kEnergyChunk) / 8;
      const uint4* row = reinterpret_cast<const uint4*>(buf[chunk & 1] + threadIdx.x * kEnergyRowBytes);
      uint4 q = row[0];
      for (int v = 0; v < nv; ++v) {
        const uint4 cur = q;
        if (v + 1 < nv) q = row[v + 1];  // next 8 values in flight during this chain
        const uint32_t w[4] = {cur.x, cur.y, cur.z, cur.w};
        double sq[8];  // x^2 of a bf16 is exact in fp64; computed off the chain
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const double a = bf16_to_f64(w[h] & 0xFFFFu);
          const double b = bf16_to_f64(w[h] >> 16);
          sq[2 * h] = __dmul_rn(a, a);
          sq[2 * h + 1] = __dmul_rn(b, b);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = __dadd_rn(acc, sq[e]);  // n ascending
      }
    }
    __syncthreads();  // buffer (chunk & 1) is refilled by the next iteration's stage()
  }
  if (threadIdx.x < nch) s[c0 + threadIdx.x] = __double2float_rn(acc);
}

// 4 consecutive elements of one row per quad (K % 4 == 0); each thread takes kQuads quads
// per pass of the grid-stride loop, their loads issued before any arithmetic.
constexpr int kQuads = 4;

__global__ void importance_kernel(const uint16_t* __restrict__ W, const float* __restrict__ s,
                                  int M, int K, float* __restrict__ I) {
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

constexpr int kMaxNoAllocDevices = 64;
std::mutex g_noalloc_mu;
float* g_noalloc_ptr[kMaxNoAllocDevices] = {};

}  // namespace

// Address of this device's static scratch, resolved once per device (the caller's current
// device is the one the call runs on).
cudaError_t noalloc_energy_scratch(float** out) {
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxNoAllocDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_energy);
    if (e != cudaSuccess) return e;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return cudaSuccess;
}

size_t importance_workspace_bytes(int K) { return ((size_t)K * sizeof(float) + 255) & ~size_t(255); }

cudaError_t launch_importance(const uint16_t* W, const uint16_t* X, int M, int K, int N,
                              float* I, float* s_scratch, cudaStream_t st) {
  channel_energy_kernel<<<(K + kEnergyChannels - 1) / kEnergyChannels, kEnergyThreads, 0, st>>>(
      X, K, N, s_scratch);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long total4 = (long long)M * K / 4;
  long long blocks = (total4 + 255) / 256;
  const long long cap = (long long)sm_count() * 8;
  if (blocks > cap) blocks = cap;
  importance_kernel<<<(unsigned)blocks, 256, 0, st>>>(W, s_scratch, M, K, I);
  return cudaGetLastError();
}

}  // namespace hinm
