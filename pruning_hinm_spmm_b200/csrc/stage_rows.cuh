// Staging of RB consecutive rows of a row-major fp32 matrix into shared memory,
// channel-major: the RB values of channel c lie contiguous at slot stage_slot(c), so one
// vector load reads a channel's RB rows.  Used by the mask (top-2 of 4 per row) and by the
// boundary search (the 2:4 bands' top-2 sums), which read the staged rows in gathered
// channel order.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "hinm_internal.h"

namespace hinm {

// Reading an ImpSrc (hinm_internal.h): the materialized I, or -- when I is null -- each
// value recomputed from W and the channel energies as fl32(fl32(w^2) s_c), the same two
// roundings as the importance kernels, so the same bits, from 2 bytes per weight instead of 4.

__device__ __forceinline__ float imp_from_w(uint32_t wbits16, float sc) {
  const float w = __uint_as_float(wbits16 << 16);
  return __fmul_rn(__fmul_rn(w, w), sc);
}

// Column c of an ImpSrc, read row by row: the channel energy is loaded once.
struct ImpColumn {
  const float* I;
  const uint16_t* W;
  float sc;
  int K, c;
  __device__ __forceinline__ float at(size_t row) const {
    if (I) return __ldg(I + row * K + c);
    return imp_from_w(__ldg(W + row * K + c), sc);
  }
};

__device__ __forceinline__ ImpColumn imp_column(const ImpSrc& q, int K, int c) {
  return ImpColumn{q.I, q.W, q.I ? 0.0f : __ldg(q.s + c), K, c};
}

// Slot of channel c (rows padded to a multiple of 8 channels): within each aligned group of
// 8 channels the 16-byte bank slot is permuted by higher bits of c, so that the strided
// channels of consecutive groups (4, 8, 16, 32 or 64 apart) fall into different banks.
__device__ __forceinline__ int stage_slot(int c) {
  return (c & ~7) | ((c ^ (c >> 3) ^ (c >> 6)) & 7);
}

template <int RB>
__device__ __forceinline__ void stage_store(float* p, const float (&v)[RB]) {
  if constexpr (RB == 8) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  } else if constexpr (RB == 4) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  } else if constexpr (RB == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
    *p = v[0];
  }
}

__device__ __forceinline__ float quad_at(const float4& q, int i) {
  return i == 0 ? q.x : (i == 1 ? q.y : (i == 2 ? q.z : q.w));
}

// src: the first of RB rows, row stride K floats (K % 4 == 0 and src 16-byte aligned, so
// every row starts on a 16-byte boundary).  NT threads; each takes quads of 4 consecutive
// channels and loads them for all RB rows, two quads per pass (2 x RB 16-byte loads in
// flight per thread) before storing them channel by channel.
template <int RB, int NT>
__device__ __forceinline__ void stage_rows(const float* __restrict__ src, int K,
                                           float* __restrict__ rows_s) {
  const int nq = K >> 2;
  for (int q0 = (int)threadIdx.x; q0 < nq; q0 += 2 * NT) {
    float4 a[2][RB];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = q0 + u * NT;
#pragma unroll
      for (int r = 0; r < RB; ++r)
        a[u][r] = q < nq ? __ldg(reinterpret_cast<const float4*>(src + (size_t)r * K) + q)
                         : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = q0 + u * NT;
      if (q < nq) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          float v[RB];
#pragma unroll
          for (int r = 0; r < RB; ++r) v[r] = quad_at(a[u][r], i);
          stage_store<RB>(rows_s + (size_t)stage_slot(4 * q + i) * RB, v);
        }
      }
    }
  }
}

// stage_rows from an ImpSrc: rows row0 .. row0 + RB - 1.  From W, each quad of 4 channels is
// one 8-byte load per row and one 16-byte load of their energies.
template <int RB, int NT>
__device__ __forceinline__ void stage_rows_imp(const ImpSrc& src, size_t row0, int K,
                                               float* __restrict__ rows_s) {
  if (src.I) {
    stage_rows<RB, NT>(src.I + row0 * K, K, rows_s);
    return;
  }
  const int nq = K >> 2;
  const uint16_t* w0 = src.W + row0 * K;
  for (int q0 = (int)threadIdx.x; q0 < nq; q0 += 2 * NT) {
    uint2 a[2][RB];
    float4 sq[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = q0 + u * NT;
      sq[u] = q < nq ? __ldg(reinterpret_cast<const float4*>(src.s) + q)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < RB; ++r)
        a[u][r] = q < nq ? __ldg(reinterpret_cast<const uint2*>(w0 + (size_t)r * K) + q)
                         : make_uint2(0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int q = q0 + u * NT;
      if (q < nq) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float sc = quad_at(sq[u], i);
          float v[RB];
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            const uint32_t word = (i < 2) ? a[u][r].x : a[u][r].y;
            v[r] = imp_from_w((i & 1) ? (word >> 16) : (word & 0xFFFFu), sc);
          }
          stage_store<RB>(rows_s + (size_t)stage_slot(4 * q + i) * RB, v);
        }
      }
    }
  }
}

}  // namespace hinm
