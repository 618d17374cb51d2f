// int8 KV-cache rows (the Atlas summary of the Gemma 4 report: int8 KV caching,
// Table 3 "+KV"): each row of head_dim values (one position, one kv head) gets
// the fp32 scale s = max|x| / 127 and the codes round-half-even(x / s) in
// [-127, 127]; a row of zeros gets s = 0 and codes 0.  Both divisions are the
// correctly rounded float32 division, so the codes are reproducible bit for bit.
//
// One warp per row, eight rows per 256-thread block; a lane holds D/32
// consecutive values (one or two 16-byte loads) and writes their codes with
// one 8- or 16-byte store.  HBM-bound: 2D bytes read, D + 4 written per row.
#include <cuda_bf16.h>

#include "gattn_internal.h"
#include "kernels/common.cuh"

namespace gattn {

namespace {

template <int D>
__global__ void __launch_bounds__(256) kv_quantize_kernel(const __nv_bfloat16* __restrict__ x,
                                                          int8_t* __restrict__ codes,
                                                          float* __restrict__ scales, long long nrows) {
  constexpr int PER = D / 32;  // values per lane
  const long long row = blockIdx.x * 8LL + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= nrows) return;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * D) + lane * (PER / 8);
  float v[PER];
#pragma unroll
  for (int i = 0; i < PER / 8; ++i) {
    const uint4 u = __ldg(src + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float2 f = unpack_bf16x2(w[j]);
      v[8 * i + 2 * j] = f.x;
      v[8 * i + 2 * j + 1] = f.y;
    }
  }
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  const float s = __fdiv_rn(amax, 127.f);
  uint32_t packed[PER / 4];
#pragma unroll
  for (int i = 0; i < PER / 4; ++i) packed[i] = 0u;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    int c = 0;
    if (s > 0.f) c = min(max(__float2int_rn(__fdiv_rn(v[i], s)), -127), 127);
    packed[i / 4] |= (static_cast<uint32_t>(c) & 0xFFu) << (8 * (i % 4));
  }
  int8_t* dst = codes + row * D + lane * PER;
  if constexpr (PER == 8)
    *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
  else
    *reinterpret_cast<uint4*>(dst) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
  if (lane == 0) scales[row] = s;
}

}  // namespace

cudaError_t launch_kv_quantize(const __nv_bfloat16* x, int8_t* codes, float* scales, long long nrows, int D,
                               cudaStream_t s) {
  if (nrows <= 0) return cudaSuccess;
  const long long blocks = (nrows + 7) / 8;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  if (D == 256) {
    kv_quantize_kernel<256><<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, codes, scales, nrows);
  } else if (D == 512) {
    kv_quantize_kernel<512><<<static_cast<unsigned>(blocks), 256, 0, s>>>(x, codes, scales, nrows);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace gattn
