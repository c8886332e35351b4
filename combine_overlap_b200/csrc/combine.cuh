// combine.cuh -- the weighted reduction of one token, shared by the stand-alone
// combine kernel (sequential mode) and the consumer role of the persistent
// kernel (overlapped mode), so both modes produce bit-identical outputs.
//
// "Fine-grained Computation-Communication Overlap via Tile-level Signaling and
// Scheduling for Mixture-of-Experts", Section 2.1, step 5 (weighted reduction):
//   out[t] = bf16( sum_{j<k} g[t][j] * y[row_of[t*k+j]] ), fp32, slot order,
// accumulated with fmaf from 0.
#pragma once

#include "common.cuh"

namespace moe {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& v, float (&f)[8]) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(u[i] << 16);
    f[2 * i + 1] = __uint_as_float(u[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&p);
}

// One warp combines token t (k <= KMAX): each pass, every lane loads U 16-byte
// vectors of each of the k rows (U*k loads in flight), then reduces them.  y rows
// are read through L2 (ld.global.cg): a row may have been written by another SM
// during this kernel.  The arithmetic per element does not depend on KMAX or U.
template <int KMAX, int U>
__device__ __forceinline__ void combine_token_warp_u(const __nv_bfloat16* __restrict__ y,
                                                     const int32_t* __restrict__ row_of,
                                                     const float* __restrict__ gate, int t, int d,
                                                     int k, __nv_bfloat16* __restrict__ out,
                                                     int lane) {
  int rows[KMAX];
  float g[KMAX];
#pragma unroll
  for (int j = 0; j < KMAX; ++j) {
    if (j < k) {
      rows[j] = row_of[(size_t)t * k + j];
      g[j] = gate[(size_t)t * k + j];
    }
  }
  const int dv = d >> 3;
  const uint4* yv = reinterpret_cast<const uint4*>(y);
  uint4* ov = reinterpret_cast<uint4*>(out) + (size_t)t * dv;
  for (int v0 = lane; v0 < dv; v0 += 32 * U) {
    uint4 in[U][KMAX];
#pragma unroll
    for (int j = 0; j < KMAX; ++j) {
      if (j < k) {
#pragma unroll
        for (int u = 0; u < U; ++u)
          if (v0 + 32 * u < dv) in[u][j] = __ldcg(yv + (size_t)rows[j] * dv + v0 + 32 * u);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (v0 + 32 * u >= dv) break;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
      for (int j = 0; j < KMAX; ++j) {
        if (j < k) {
          float f[8];
          bf16x8_to_f32(in[u][j], f);
#pragma unroll
          for (int i = 0; i < 8; ++i) acc[i] = fmaf(g[j], f[i], acc[i]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(acc[0], acc[1]);
      o.y = pack_bf16x2(acc[2], acc[3]);
      o.z = pack_bf16x2(acc[4], acc[5]);
      o.w = pack_bf16x2(acc[6], acc[7]);
      ov[v0 + 32 * u] = o;
    }
  }
}

// The combine kernels' form: two vectors per lane per pass, any k <= MAX_K.
__device__ __forceinline__ void combine_token_warp(const __nv_bfloat16* __restrict__ y,
                                                   const int32_t* __restrict__ row_of,
                                                   const float* __restrict__ gate, int t, int d,
                                                   int k, __nv_bfloat16* __restrict__ out,
                                                   int lane) {
  combine_token_warp_u<MAX_K, 2>(y, row_of, gate, t, d, k, out, lane);
}

}  // namespace moe
