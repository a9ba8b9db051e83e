// Hard-Concrete soft 2:4 mask, forward (FlexHiNM-GP notes, 关键设计 3: the binary mask of
// each group of 4 parameterised by learnable logits log alpha; with noise eps ~ U(0, 1),
// s = sigmoid((log eps - log(1 - eps) + log alpha) / tau), stretched to (-0.1, 1.1) and
// clipped to [0, 1]; regularisers mean(z) and mean over groups of |sum z - 2|; hardened at
// 0.5).  The noise is an input: eps = 1/2 everywhere gives the deterministic mask.
//
// One HBM stream: a thread per group of 4 (16-byte loads of log alpha and eps, a 16-byte
// store of z and a 4-byte store of the hardened bits), kHcUnroll groups in flight per thread,
// grid-stride; the two regulariser sums in fp64, block-reduced, one atomic add per block.
// The fp32 arithmetic calls CUDA's logf and expf.
#include <cuda_runtime.h>

#include "hinm_internal.h"

namespace hinm {
namespace {

constexpr int kHcThreads = 256;
constexpr int kHcUnroll = 4;
constexpr float kHcLow = -0.1f, kHcHigh = 1.1f;  // the stretch interval

int hc_sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// inv_tau = fl32(1 / tau); the reciprocals are the correctly rounded ones.  The noise logit
// log(eps / (1 - eps)) takes one logf of the ratio (three fp32 roundings: 1 - eps, its
// reciprocal, the product; eps = 0 or 1 still give -inf / +inf).
__device__ __forceinline__ float hc_z(float la, float e, float inv_tau) {
  const float logit = logf(__fmul_rn(e, __frcp_rn(__fsub_rn(1.0f, e))));
  const float x = __fmul_rn(__fadd_rn(logit, la), inv_tau);
  const float s = __frcp_rn(__fadd_rn(1.0f, expf(-x)));
  const float sb = __fadd_rn(__fmul_rn(s, __fsub_rn(kHcHigh, kHcLow)), kHcLow);
  // clip to [0, 1] by comparisons, so that a NaN (a NaN input, or -inf + inf in the logit)
  // passes through as NaN; fminf / fmaxf would return the non-NaN operand
  return sb < 0.0f ? 0.0f : (sb > 1.0f ? 1.0f : sb);
}

__global__ void __launch_bounds__(kHcThreads) hard_concrete_kernel(
    const float4* __restrict__ log_alpha, const float4* __restrict__ eps, long long ngroups,
    float tau, float4* __restrict__ z, uchar4* __restrict__ hard, double* __restrict__ sums) {
  __shared__ double red[2][kHcThreads / 32];
  double acc_z = 0.0, acc_h = 0.0;
  const float inv_tau = __frcp_rn(tau);
  const long long stride = (long long)gridDim.x * blockDim.x;
  for (long long g0 = blockIdx.x * (long long)blockDim.x + threadIdx.x; g0 < ngroups;
       g0 += stride * kHcUnroll) {
    float4 a[kHcUnroll], e[kHcUnroll];
#pragma unroll
    for (int u = 0; u < kHcUnroll; ++u) {
      const long long g = g0 + u * stride;
      if (g < ngroups) {
        a[u] = __ldg(log_alpha + g);
        e[u] = __ldg(eps + g);
      }
    }
#pragma unroll
    for (int u = 0; u < kHcUnroll; ++u) {
      const long long g = g0 + u * stride;
      if (g >= ngroups) break;
      float4 o;
      o.x = hc_z(a[u].x, e[u].x, inv_tau);
      o.y = hc_z(a[u].y, e[u].y, inv_tau);
      o.z = hc_z(a[u].z, e[u].z, inv_tau);
      o.w = hc_z(a[u].w, e[u].w, inv_tau);
      __stcs(z + g, o);
      if (hard)
        hard[g] = make_uchar4(o.x > 0.5f, o.y > 0.5f, o.z > 0.5f, o.w > 0.5f);
      const double gs = (double)o.x + (double)o.y + (double)o.z + (double)o.w;
      acc_z += gs;
      acc_h += fabs(gs - 2.0);
    }
  }
  if (!sums) return;
  for (int o = 16; o > 0; o >>= 1) {
    acc_z += __shfl_xor_sync(0xffffffffu, acc_z, o);
    acc_h += __shfl_xor_sync(0xffffffffu, acc_h, o);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) {
    red[0][warp] = acc_z;
    red[1][warp] = acc_h;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double tz = 0.0, th = 0.0;
    for (int w = 0; w < kHcThreads / 32; ++w) {
      tz += red[0][w];
      th += red[1][w];
    }
    atomicAdd(sums, tz);
    atomicAdd(sums + 1, th);
  }
}

}  // namespace

cudaError_t launch_hard_concrete(const float* log_alpha, const float* eps, long long n, float tau,
                                 float* z, uint8_t* hard, double* sums, cudaStream_t s) {
  const long long ng = n / 4;
  if (sums) {
    cudaError_t e = cudaMemsetAsync(sums, 0, 2 * sizeof(double), s);
    if (e != cudaSuccess) return e;
  }
  long long blocks = (ng + kHcThreads - 1) / kHcThreads;
  const long long cap = (long long)hc_sm_count() * 8;
  if (blocks > cap) blocks = cap;
  hard_concrete_kernel<<<(unsigned)blocks, kHcThreads, 0, s>>>(
      reinterpret_cast<const float4*>(log_alpha), reinterpret_cast<const float4*>(eps), ng, tau,
      reinterpret_cast<float4*>(z), reinterpret_cast<uchar4*>(hard), sums);
  return cudaGetLastError();
}

}  // namespace hinm
