// Warp-per-row helpers for the QK-norm + RoPE prologue (sm_100a).
//
// A warp holds one head row of D = 256 * NCH dims; lane l owns the 8-dim
// chunks c = l + 32 i (i < NCH), dims [8c, 8c + 8).  Used by the key prologue,
// the decode query/key prologues and the prefill query prologue.
#pragma once

#include <cuda_bf16.h>

#include "gattn_internal.h"
#include "kernels/common.cuh"

namespace gattn {

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <int NCH>
__device__ __forceinline__ void load_row(const __nv_bfloat16* row, int lane, float (&x)[NCH][8]) {
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(row) + lane + 32 * i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = unpack_bf16x2(w[e]);
      x[i][2 * e] = f.x;
      x[i][2 * e + 1] = f.y;
    }
  }
}

// The same chunks from an int8 row, dequantised by the row's scale.
template <int NCH>
__device__ __forceinline__ void load_row_q8(const int8_t* row, float scale, int lane, float (&x)[NCH][8]) {
#pragma unroll
  for (int i = 0; i < NCH; ++i) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(row) + lane + 32 * i);
    float2 c[4];
    unpack_i8x4(u.x, c[0], c[1]);
    unpack_i8x4(u.y, c[2], c[3]);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[i][2 * e] = c[e].x * scale;
      x[i][2 * e + 1] = c[e].y * scale;
    }
  }
}

__device__ __forceinline__ int checked_pos(int pos, const LayerArgs& la, uint32_t* status) {
  if (pos < 0 || pos >= la.rope_max_pos) {
    flag_status(status, kStatusBounds);
    return pos < 0 ? 0 : la.rope_max_pos - 1;
  }
  return pos;
}

// RMSNorm (optional) then RoPE (optional) on a warp-held row, in fp32.
template <int NCH>
__device__ __forceinline__ void transform_row(float (&x)[NCH][8], int lane, int pos,
                                              const LayerArgs& la, const float* w,
                                              uint32_t* status) {
  constexpr int D = NCH * 256;
  if (la.qk_norm) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += x[i][e] * x[i][e];
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / static_cast<float>(D) + la.eps);
    const float off = la.qk_norm == 1 ? 1.f : 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const int d = 8 * (lane + 32 * i) + e;
        x[i][e] = x[i][e] * r * (__ldg(w + d) + off);
      }
  }
  if (la.rot > 0) {
    pos = checked_pos(pos, la, status);
    const int half = la.rot >> 1;
    const int h16 = la.rot >> 4;  // chunks in half the rotated slice
    float pr[NCH][8];
    if (h16 < 32) {
#pragma unroll
      for (int i = 0; i < NCH; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) pr[i][e] = __shfl_xor_sync(0xffffffffu, x[i][e], h16);
    } else {
      // rotated slice of 512 dims: the partner chunk is this lane's other chunk
#pragma unroll
      for (int i = 0; i < NCH; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) pr[i][e] = x[NCH - 1 - i][e];
    }
    const float2* trow = la.rope_tab + static_cast<size_t>(pos) * half;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = lane + 32 * i;
      if (8 * c < la.rot) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int d = 8 * c + e;
          const bool first = d < half;
          const float2 cs = __ldg(trow + (first ? d : d - half));
          x[i][e] = first ? x[i][e] * cs.x - pr[i][e] * cs.y : x[i][e] * cs.x + pr[i][e] * cs.y;
        }
      }
    }
  }
}

// The same RMSNorm + RoPE with the (cos, sin) of each of the lane's elements
// given (cs[i][e] for dim 8 (lane + 32 i) + e, read only on rotated dims):
// rows that share a position share the angles.
template <int NCH>
__device__ __forceinline__ void transform_row_cs(float (&x)[NCH][8], int lane, const LayerArgs& la,
                                                 const float* w, const float2 (&cs)[NCH][8]) {
  constexpr int D = NCH * 256;
  if (la.qk_norm) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) ss += x[i][e] * x[i][e];
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / static_cast<float>(D) + la.eps);
    const float off = la.qk_norm == 1 ? 1.f : 0.f;
    const float4* w4 = reinterpret_cast<const float4*>(w);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = lane + 32 * i;
      const float4 g0 = __ldg(w4 + 2 * c), g1 = __ldg(w4 + 2 * c + 1);
      x[i][0] *= r * (g0.x + off); x[i][1] *= r * (g0.y + off);
      x[i][2] *= r * (g0.z + off); x[i][3] *= r * (g0.w + off);
      x[i][4] *= r * (g1.x + off); x[i][5] *= r * (g1.y + off);
      x[i][6] *= r * (g1.z + off); x[i][7] *= r * (g1.w + off);
    }
  }
  if (la.rot > 0) {
    const int half = la.rot >> 1;
    const int h16 = la.rot >> 4;
    float pr[NCH][8];
    if (h16 < 32) {
#pragma unroll
      for (int i = 0; i < NCH; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) pr[i][e] = __shfl_xor_sync(0xffffffffu, x[i][e], h16);
    } else {
#pragma unroll
      for (int i = 0; i < NCH; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) pr[i][e] = x[NCH - 1 - i][e];
    }
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = lane + 32 * i;
      if (8 * c < la.rot) {
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const bool first = 8 * c + e < half;
          x[i][e] = first ? x[i][e] * cs[i][e].x - pr[i][e] * cs[i][e].y
                          : x[i][e] * cs[i][e].x + pr[i][e] * cs[i][e].y;
        }
      }
    }
  }
}

// 8 floats <-> 8 packed bf16 (16 bytes)
__device__ __forceinline__ void unpack8(const uint4 u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = unpack_bf16x2(w[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}
__device__ __forceinline__ uint4 pack8(const float (&x)[8]) {
  uint4 u;
  u.x = pack_bf16x2(x[0], x[1]);
  u.y = pack_bf16x2(x[2], x[3]);
  u.z = pack_bf16x2(x[4], x[5]);
  u.w = pack_bf16x2(x[6], x[7]);
  return u;
}

// 16-byte chunk c (8 dims) of row r of a tile held in shared memory as
// 128-byte swizzled 64-dim slabs of slab_bytes each (the TMA layout).
__device__ __forceinline__ uint4* tile_chunk(uint8_t* tile, int slab_bytes, int r, int c) {
  return reinterpret_cast<uint4*>(tile + (c >> 3) * slab_bytes + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

}  // namespace gattn
