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

// One thread per channel c: sequential fp64 sum over n = 0..N-1 (N % 8 == 0).  Up to 8
// 16-byte loads are in flight before they are summed, in order.
__global__ void channel_energy_kernel(const uint16_t* __restrict__ X, int K, int N,
                                      float* __restrict__ s) {
  const int c = blockIdx.x * blockDim.x + threadIdx.x;
  if (c >= K) return;
  const uint4* row = reinterpret_cast<const uint4*>(X + (size_t)c * N);
  double acc = 0.0;
  const int nv = N / 8;
  constexpr int kBatch = 8;
  int v0 = 0;
  for (; v0 + kBatch <= nv; v0 += kBatch) {
    uint4 q[kBatch];
#pragma unroll
    for (int k = 0; k < kBatch; ++k) q[k] = __ldg(row + v0 + k);
#pragma unroll
    for (int k = 0; k < kBatch; ++k) {
      const uint32_t w[4] = {q[k].x, q[k].y, q[k].z, q[k].w};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        const double a = bf16_to_f64(w[h] & 0xFFFFu);
        const double b = bf16_to_f64(w[h] >> 16);
        acc = __dadd_rn(acc, __dmul_rn(a, a));  // x^2 of a bf16 is exact in fp64
        acc = __dadd_rn(acc, __dmul_rn(b, b));
      }
    }
  }
  for (; v0 < nv; ++v0) {
    const uint4 q = __ldg(row + v0);
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const double a = bf16_to_f64(w[h] & 0xFFFFu);
      const double b = bf16_to_f64(w[h] >> 16);
      acc = __dadd_rn(acc, __dmul_rn(a, a));
      acc = __dadd_rn(acc, __dmul_rn(b, b));
    }
  }
  s[c] = __double2float_rn(acc);
}

// 4 consecutive elements of one row per thread (K % 4 == 0).
__global__ void importance_kernel(const uint16_t* __restrict__ W, const float* __restrict__ s,
                                  int M, int K, float* __restrict__ I) {
  const long long total4 = (long long)M * K / 4;
  const int k4 = K / 4;
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < total4;
       q += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(q % k4) * 4;
    const uint2 wv = __ldg(reinterpret_cast<const uint2*>(W) + q);
    const float4 sv = __ldg(reinterpret_cast<const float4*>(s + c));
    const float w0 = __uint_as_float(wv.x << 16), w1 = __uint_as_float(wv.x & 0xFFFF0000u);
    const float w2 = __uint_as_float(wv.y << 16), w3 = __uint_as_float(wv.y & 0xFFFF0000u);
    float4 o;
    o.x = __fmul_rn(__fmul_rn(w0, w0), sv.x);
    o.y = __fmul_rn(__fmul_rn(w1, w1), sv.y);
    o.z = __fmul_rn(__fmul_rn(w2, w2), sv.z);
    o.w = __fmul_rn(__fmul_rn(w3, w3), sv.w);
    __stcs(reinterpret_cast<float4*>(I) + q, o);
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
  channel_energy_kernel<<<(K + 63) / 64, 64, 0, st>>>(X, K, N, s_scratch);
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
