// RoPE table, key prologue (QK-norm + RoPE) and the split-KV decode kernels.
//
// Decode follows the layer definition of the Gemma model cards for one new
// token: the query at position L-1 attends over cache rows [0, L) (the last
// `window` of them on sliding-window layers), keys pass through QK-norm and
// RoPE at their own positions, and with K=V the raw cached keys are the
// values (KerasFormers "Gemma 4", What changed).  The cache read is split in
// chunks across CTAs; each CTA writes a (max, sum, weighted-sum) partial and a
// second kernel merges them with the log-sum-exp rule.
#include <cuda_bf16.h>

#include <cstdio>
#include <mutex>

#include "gattn_internal.h"
#include "kernels/common.cuh"
#include "kernels/rowops.cuh"

namespace gattn {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------------------
// RoPE table: tab[p][t] = (cos, sin)(p * theta^(-2t/F)), angle in double.
// ---------------------------------------------------------------------------
__global__ void rope_table_kernel(float2* tab, double theta, int half, int freq_dim,
                                  long long total) {
  long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= total) return;
  const int p = static_cast<int>(i / half);
  const int t = static_cast<int>(i % half);
  const double inv_freq = pow(theta, -2.0 * t / static_cast<double>(freq_dim));
  double sn, cs;
  sincos(static_cast<double>(p) * inv_freq, &sn, &cs);
  tab[i] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
}

cudaError_t launch_rope_table(float2* tab, double theta, int half, int freq_dim, int max_pos,
                              cudaStream_t s) {
  const long long total = static_cast<long long>(max_pos) * half;
  const int threads = 256;
  const long long blocks = (total + threads - 1) / threads;
  rope_table_kernel<<<static_cast<unsigned>(blocks), threads, 0, s>>>(tab, theta, half, freq_dim,
                                                                      total);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Query and key prologue for prefill, elementwise.  TPR = D/16 threads (a 16-
// or 32-lane group) serve one token (b, s); thread i owns two 8-dim chunks of
// every row of the token: a RoPE pair (chunk i and chunk i + R/16) when
// i < R/16, else two unrotated chunks.  It reads the token's position and
// its (cos, sin) from the RoPE table once, then walks the token's H query
// rows (query gain) and Hkv key rows (key gain), RB rows at a time with
// their loads issued together; outputs keep the input layouts.
// ---------------------------------------------------------------------------
// MODE 0: a prompt's queries and keys, positions from `positions`.  MODE 1: a
// chunk's queries only (token bs = b * C + s at position prefix[b] + s).
// MODE 2: a cache's keys only (token bs = b * max_len + s at position s),
// skipping the rows past the chunk (s >= prefix[b] + C).  MODE 3: a chunk's new
// keys only (token bs = b * C + s at position prefix[b] + s), written to cache
// row prefix[b] + s of kt (a transformed cache's append).
struct ChunkPrep {
  const int* prefix;
  int C, max_len;
};

template <int TPR, int RB, int MODE>
__global__ void __launch_bounds__(256) qkprep_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k,
                                                     const int* __restrict__ positions,
                                                     bf16* __restrict__ qt, bf16* __restrict__ kt,
                                                     long long tokens, LayerArgs la, uint32_t* status,
                                                     ChunkPrep cp) {
  constexpr int D = TPR * 16;
  pdl_launch_dependents();  // the attention kernel may be scheduled now; it waits for this grid
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long bs = gid / TPR;
  const int i = static_cast<int>(gid % TPR);
  if (bs >= tokens) return;  // whole groups leave together (TPR divides 32)
  int tok_pos = 0;
  long long kdst = bs;  // output row (token) of the key rows
  if constexpr (MODE == 0) {
    tok_pos = positions ? __ldg(positions + bs) : 0;
  } else {
    const int per = MODE == 2 ? cp.max_len : cp.C;
    const int b = static_cast<int>(bs / per), s = static_cast<int>(bs % per);
    const int pre = min(max(__ldg(cp.prefix + b), 0), cp.max_len - cp.C);
    if (MODE == 2 && s >= pre + cp.C) return;  // a cache row no query of the chunk sees
    tok_pos = MODE == 2 ? s : pre + s;
    if (MODE == 3) kdst = static_cast<long long>(b) * cp.max_len + pre + s;
  }
  const unsigned gmask = TPR == 32 ? 0xffffffffu : (0xffffu << (threadIdx.x & 16));
  const int h8 = la.rot >> 4;  // chunks in half the rotated slice
  const bool rotated = i < h8;
  const int c0 = rotated ? i : 2 * h8 + 2 * (i - h8);
  const int c1 = rotated ? i + h8 : c0 + 1;
  float4 cs[4];  // (cos, sin) of pairs 8i .. 8i+7, two pairs per float4
  if (rotated) {
    const int pos = checked_pos(tok_pos, la, status);
    const float4* trow = reinterpret_cast<const float4*>(la.rope_tab + static_cast<size_t>(pos) * (la.rot >> 1)) + 4 * i;
#pragma unroll
    for (int e = 0; e < 4; ++e) cs[e] = __ldg(trow + e);
  }
  const float off = la.qk_norm == 1 ? 1.f : 0.f;
  const int nq = MODE >= 2 ? 0 : la.H;  // query rows of the token, then key rows
  const int nrows = nq + (MODE == 1 ? 0 : la.Hkv);
  for (int r0 = 0; r0 < nrows; r0 += RB) {
    uint4 u0[RB], u1[RB];
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      const int r = r0 + u;
      if (r < nrows) {
        const uint4* src = reinterpret_cast<const uint4*>(
            r < nq ? q + (bs * la.H + r) * D : k + (bs * la.Hkv + (r - nq)) * D);
        u0[u] = __ldg(src + c0);
        u1[u] = __ldg(src + c1);
      }
    }
#pragma unroll
    for (int u = 0; u < RB; ++u) {
      const int r = r0 + u;
      if (r >= nrows) break;  // uniform over the group
      const bool is_q = r < nq;
      float x0[8], x1[8];
      unpack8(u0[u], x0);
      unpack8(u1[u], x1);
      if (la.qk_norm) {
        float ss = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) ss = fmaf(x0[e], x0[e], fmaf(x1[e], x1[e], ss));
#pragma unroll
        for (int o = TPR / 2; o > 0; o >>= 1) ss += __shfl_xor_sync(gmask, ss, o);
        const float rn = rsqrtf(ss / static_cast<float>(D) + la.eps);
        const float4* w4 = reinterpret_cast<const float4*>(is_q ? la.q_norm_w : la.k_norm_w);
        const float4 a0 = __ldg(w4 + 2 * c0), a1 = __ldg(w4 + 2 * c0 + 1);
        const float4 b0 = __ldg(w4 + 2 * c1), b1 = __ldg(w4 + 2 * c1 + 1);
        x0[0] *= rn * (a0.x + off); x0[1] *= rn * (a0.y + off); x0[2] *= rn * (a0.z + off); x0[3] *= rn * (a0.w + off);
        x0[4] *= rn * (a1.x + off); x0[5] *= rn * (a1.y + off); x0[6] *= rn * (a1.z + off); x0[7] *= rn * (a1.w + off);
        x1[0] *= rn * (b0.x + off); x1[1] *= rn * (b0.y + off); x1[2] *= rn * (b0.z + off); x1[3] *= rn * (b0.w + off);
        x1[4] *= rn * (b1.x + off); x1[5] *= rn * (b1.y + off); x1[6] *= rn * (b1.z + off); x1[7] *= rn * (b1.w + off);
      }
      if (rotated) {
#pragma unroll
        for (int e = 0; e < 8; e += 2) {
          const float4 c = cs[e / 2];
          const float a = x0[e], bb = x1[e], a2 = x0[e + 1], b2 = x1[e + 1];
          x0[e] = a * c.x - bb * c.y;
          x1[e] = bb * c.x + a * c.y;
          x0[e + 1] = a2 * c.z - b2 * c.w;
          x1[e + 1] = b2 * c.z + a2 * c.w;
        }
      }
      uint4* dst = reinterpret_cast<uint4*>(is_q ? qt + (bs * la.H + r) * D : kt + (kdst * la.Hkv + (r - nq)) * D);
      dst[c0] = pack8(x0);
      dst[c1] = pack8(x1);
    }
  }
}

cudaError_t launch_qkprep(const bf16* q, const bf16* k, const int* positions, bf16* qt, bf16* kt,
                          int B, int S, const LayerArgs& la, uint32_t* status, cudaStream_t s) {
  const long long tokens = static_cast<long long>(B) * S;
  const long long threads = tokens * (la.D / 16);
  const unsigned blocks = static_cast<unsigned>((threads + 255) / 256);
  const ChunkPrep cp{nullptr, 0, 0};
  if (la.D == 256)
    qkprep_kernel<16, 3, 0><<<blocks, 256, 0, s>>>(q, k, positions, qt, kt, tokens, la, status, cp);
  else
    qkprep_kernel<32, 3, 0><<<blocks, 256, 0, s>>>(q, k, positions, qt, kt, tokens, la, status, cp);
  return cudaGetLastError();
}

cudaError_t launch_qkprep_chunk(const bf16* q, const bf16* k_cache, const int* prefix, bf16* qt, bf16* kt,
                                int B, int C, int max_len, const LayerArgs& la, uint32_t* status,
                                cudaStream_t s, bool with_keys) {
  const ChunkPrep cp{prefix, C, max_len};
  const long long tq = static_cast<long long>(B) * C, tk = static_cast<long long>(B) * max_len;
  const unsigned bq = static_cast<unsigned>((tq * (la.D / 16) + 255) / 256);
  const unsigned bk = static_cast<unsigned>((tk * (la.D / 16) + 255) / 256);
  if (la.D == 256) {
    if (with_keys) qkprep_kernel<16, 3, 2><<<bk, 256, 0, s>>>(nullptr, k_cache, nullptr, nullptr, kt, tk, la, status, cp);
    qkprep_kernel<16, 3, 1><<<bq, 256, 0, s>>>(q, nullptr, nullptr, qt, nullptr, tq, la, status, cp);
  } else {
    if (with_keys) qkprep_kernel<32, 3, 2><<<bk, 256, 0, s>>>(nullptr, k_cache, nullptr, nullptr, kt, tk, la, status, cp);
    qkprep_kernel<32, 3, 1><<<bq, 256, 0, s>>>(q, nullptr, nullptr, qt, nullptr, tq, la, status, cp);
  }
  return cudaGetLastError();
}

cudaError_t launch_key_append_transformed(const bf16* k_new, bf16* k_cache, const int* prefix, int B, int C,
                                          int max_len, const LayerArgs& la, uint32_t* status, cudaStream_t s) {
  const ChunkPrep cp{prefix, C, max_len};
  const long long tk = static_cast<long long>(B) * C;
  const unsigned bk = static_cast<unsigned>((tk * (la.D / 16) + 255) / 256);
  if (la.D == 256)
    qkprep_kernel<16, 3, 3><<<bk, 256, 0, s>>>(nullptr, k_new, nullptr, nullptr, k_cache, tk, la, status, cp);
  else
    qkprep_kernel<32, 3, 3><<<bk, 256, 0, s>>>(nullptr, k_new, nullptr, nullptr, k_cache, tk, la, status, cp);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Cache append: row (b, s, h) of the new rows to cache row (b, prefix[b] + s, h),
// one 16-byte word per thread.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) kv_append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                                        uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                                        const int* __restrict__ prefix, int C, int max_len,
                                                        int row_words, long long words, uint32_t* status) {
  const long long gid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= words) return;
  const long long per_b = static_cast<long long>(C) * row_words;  // words of one sequence's new rows
  // (k_new null: values only, the keys being written transformed by the prologue kernel)
  const int b = static_cast<int>(gid / per_b);
  const long long w = gid % per_b;
  const int raw = __ldg(prefix + b);
  const int pre = min(max(raw, 0), max_len - C);
  if (w == 0 && pre != raw && status) flag_status(status, kStatusBounds);
  const long long dst = (static_cast<long long>(b) * max_len + pre) * row_words + w;
  if (k_new) k_cache[dst] = __ldg(k_new + gid);
  if (v_new) v_cache[dst] = __ldg(v_new + gid);
}

cudaError_t launch_kv_append(const bf16* k_new, const bf16* v_new, bf16* k_cache, bf16* v_cache,
                             const int* prefix, int B, int C, int max_len, int Hkv, int D, uint32_t* status,
                             cudaStream_t s) {
  const int row_words = Hkv * D / 8;  // one position's kv heads, in 16-byte words
  const long long words = static_cast<long long>(B) * C * row_words;
  if (words <= 0) return cudaSuccess;
  const long long blocks = (words + 255) / 256;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidValue;
  kv_append_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(k_new), reinterpret_cast<const uint4*>(v_new), reinterpret_cast<uint4*>(k_cache),
      reinterpret_cast<uint4*>(v_cache), prefix, C, max_len, row_words, words, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Split-KV decode.  CTA = (split, kv head, b); NW warps.  Warp w serves the
// head group hg = w % NHG (HPW query heads) and the key lane kg = w / NHG,
// striding over the chunk's keys by KW = NW / NHG.
// ---------------------------------------------------------------------------
constexpr int kDecodeWarps = 4;

template <int NCH, int HPW>
__global__ void __launch_bounds__(kDecodeWarps * 32) decode_split_kernel(DecodeArgs da,
                                                                          LayerArgs la) {
  constexpr int D = NCH * 256;
  constexpr int NW = kDecodeWarps;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = la.G;
  const int NHG = G / HPW;
  const int KW = NW / NHG;
  extern __shared__ float smem[];
  float* qt = smem;                 // [G][D]
  float* pm = qt + G * D;           // [NW][HPW]
  float* pl = pm + NW * HPW;        // [NW][HPW]
  float* po = pl + NW * HPW;        // [NW][HPW][D]

  const size_t head0 = static_cast<size_t>(b) * la.H + static_cast<size_t>(kvh) * G;
  const int L = __ldg(da.seq_lens + b);
  const int lo = (L >= 1 && la.window > 0) ? max(0, L - la.window) : 0;
  const int start = lo + split * da.chunk;
  const int end = min(L, start + da.chunk);
  if (L < 1 || L > da.max_len || start >= end) {
    if (L < 1 || L > da.max_len) {
      if (threadIdx.x == 0 && split == 0 && kvh == 0) flag_status(da.status, kStatusBounds);
    }
    for (int h = threadIdx.x; h < G; h += blockDim.x) {
      float* ml = da.part_ml + ((head0 + h) * da.nsplit + split) * 2;
      ml[0] = -INFINITY;
      ml[1] = 0.f;
    }
    return;
  }

  // query prologue: norm, rope at position L-1, fold scale*log2(e)
  for (int h = warp; h < G; h += NW) {
    float x[NCH][8];
    load_row<NCH>(da.q + (head0 + h) * D, lane, x);
    transform_row<NCH>(x, lane, L - 1, la, la.q_norm_w, da.status);
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) qt[h * D + 8 * (lane + 32 * i) + e] = x[i][e] * la.scale_log2;
  }
  __syncthreads();

  const int hg = warp % NHG, kg = warp / NHG;
  float qreg[HPW][NCH][8];
#pragma unroll
  for (int hh = 0; hh < HPW; ++hh)
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) qreg[hh][i][e] = qt[(hg * HPW + hh) * D + 8 * (lane + 32 * i) + e];

  float o[HPW][NCH][8];
  float m[HPW], l[HPW];
#pragma unroll
  for (int hh = 0; hh < HPW; ++hh) {
    m[hh] = -INFINITY;
    l[hh] = 0.f;
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) o[hh][i][e] = 0.f;
  }
  const float log2e_cap = la.softcap > 0.f ? 1.4426950408889634f : 0.f;

  for (int j = start + kg; j < end; j += KW) {
    const size_t rowidx = (static_cast<size_t>(b) * da.max_len + j) * la.Hkv + kvh;  // (position, kv head)
    const size_t rowoff = rowidx * D;
    float kr[NCH][8];
    if (da.kq) load_row_q8<NCH>(da.kq + rowoff, __ldg(da.ks + rowidx), lane, kr);  // an int8 cache
    else load_row<NCH>(da.k + rowoff, lane, kr);
    float kx[NCH][8];
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) kx[i][e] = kr[i][e];
    if (!la.kt_cache) transform_row<NCH>(kx, lane, j, la, la.k_norm_w, da.status);
    float s[HPW];
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) {
      float acc = 0.f;
#pragma unroll
      for (int i = 0; i < NCH; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc = fmaf(qreg[hh][i][e], kx[i][e], acc);
      s[hh] = warp_sum(acc);
      if (la.softcap > 0.f) {
        // logits are in log2 units here: cap the natural-unit value c*tanh(x/c)
        const float nat = s[hh] / 1.4426950408889634f;
        s[hh] = la.softcap * tanhf(nat / la.softcap) * log2e_cap;
      }
    }
    if (!la.k_eq_v) {
      if (da.kq) load_row_q8<NCH>(da.vq + rowoff, __ldg(da.vs + rowidx), lane, kr);
      else load_row<NCH>(da.v + rowoff, lane, kr);
    }
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) {
      const float mn = fmaxf(m[hh], s[hh]);
      const float alpha = ex2(m[hh] - mn);
      const float p = ex2(s[hh] - mn);
      l[hh] = l[hh] * alpha + p;
#pragma unroll
      for (int i = 0; i < NCH; ++i)
#pragma unroll
        for (int e = 0; e < 8; ++e) o[hh][i][e] = fmaf(o[hh][i][e], alpha, p * kr[i][e]);
      m[hh] = mn;
    }
  }

#pragma unroll
  for (int hh = 0; hh < HPW; ++hh) {
    if (lane == 0) {
      pm[warp * HPW + hh] = m[hh];
      pl[warp * HPW + hh] = l[hh];
    }
#pragma unroll
    for (int i = 0; i < NCH; ++i)
#pragma unroll
      for (int e = 0; e < 8; ++e) po[(warp * HPW + hh) * D + 8 * (lane + 32 * i) + e] = o[hh][i][e];
  }
  __syncthreads();

  // merge the KW key lanes of each head, write this CTA's partial
  for (int idx = threadIdx.x; idx < G * D; idx += NW * 32) {
    const int h = idx / D, d = idx % D;
    const int g = h / HPW, hh = h % HPW;
    float M = -INFINITY;
    for (int k2 = 0; k2 < KW; ++k2) M = fmaxf(M, pm[(k2 * NHG + g) * HPW + hh]);
    float num = 0.f, den = 0.f;
    for (int k2 = 0; k2 < KW; ++k2) {
      const int wi = (k2 * NHG + g) * HPW + hh;
      const float lw = pl[wi];
      if (lw > 0.f) {
        const float f = ex2(pm[wi] - M);
        num += f * po[wi * D + d];
        den += f * lw;
      }
    }
    const size_t slot = (head0 + h) * da.nsplit + split;
    da.part_o[slot * D + d] = num;
    if (d == 0) {
      da.part_ml[slot * 2] = M;
      da.part_ml[slot * 2 + 1] = den;
    }
  }
}

// Merge the per-chunk partials of one (b, h) row: M = max of the partials'
// maxima, weights 2^(m_c - M) (0 for empty partials), o = sum_c w_c O_c /
// sum_c w_c l_c.  The (m, l) pairs are read by all threads at once and reduced
// through shared memory; only partials with a non-zero weight are read.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(DecodeArgs da, LayerArgs la) {
  constexpr int PER = D / 128;
  extern __shared__ float wsm[];  // [nsplit] weights, then [8] reduction scratch
  float* red = wsm + da.nsplit;
  pdl_wait();  // the split kernel's partials are complete and visible past here
  const int h = blockIdx.x, b = blockIdx.y;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const size_t base = (static_cast<size_t>(b) * la.H + h) * da.nsplit;
  float mloc = -INFINITY;
  for (int s = t; s < da.nsplit; s += 128) {
    const float2 ml = *reinterpret_cast<const float2*>(da.part_ml + (base + s) * 2);
    if (ml.y > 0.f) mloc = fmaxf(mloc, ml.x);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(0xffffffffu, mloc, o));
  if (lane == 0) red[warp] = mloc;
  __syncthreads();
  const float M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  float dloc = 0.f;
  for (int s = t; s < da.nsplit; s += 128) {
    const float2 ml = *reinterpret_cast<const float2*>(da.part_ml + (base + s) * 2);
    const float f = ml.y > 0.f ? ex2(ml.x - M) : 0.f;
    wsm[s] = f;
    dloc += f * ml.y;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dloc += __shfl_xor_sync(0xffffffffu, dloc, o);
  if (lane == 0) red[4 + warp] = dloc;
  __syncthreads();
  const float den = (red[4] + red[5]) + (red[6] + red[7]);
  float num[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) num[e] = 0.f;
  for (int s = 0; s < da.nsplit; ++s) {
    const float f = wsm[s];
    if (f == 0.f) continue;  // uniform over the block
    const float* src = da.part_o + (base + s) * D + t * PER;
    if constexpr (PER == 2) {
      const float2 v = *reinterpret_cast<const float2*>(src);
      num[0] = fmaf(f, v.x, num[0]);
      num[1] = fmaf(f, v.y, num[1]);
    } else {
#pragma unroll
      for (int e = 0; e < PER; e += 4) {
        const float4 v = *reinterpret_cast<const float4*>(src + e);
        num[e] = fmaf(f, v.x, num[e]);
        num[e + 1] = fmaf(f, v.y, num[e + 1]);
        num[e + 2] = fmaf(f, v.z, num[e + 2]);
        num[e + 3] = fmaf(f, v.w, num[e + 3]);
      }
    }
  }
  const float inv = den > 0.f ? 1.f / den : 0.f;
  bf16* dst = da.out + (static_cast<size_t>(b) * la.H + h) * D + t * PER;
#pragma unroll
  for (int e = 0; e < PER; e += 2) {
    *reinterpret_cast<uint32_t*>(dst + e) = pack_bf16x2(num[e] * inv, num[e + 1] * inv);
  }
}

void decode_plan(const LayerArgs& la, int B, int max_len, int* nsplit, int* chunk, int max_split) {
  if (!decode_tc_supported(la) && decode_simt_supported(la)) {
    decode_simt_plan(la, B, max_len, max_split, nsplit, chunk);
    return;
  }
  const int span = la.window > 0 ? (la.window < max_len ? la.window : max_len) : max_len;
  int c = la.window > 0 ? 256 : 2048;
  if ((span + c - 1) / c > max_split && max_split > 0) c = (span + max_split - 1) / max_split;
  *chunk = c;
  *nsplit = (span + c - 1) / c;
}

template <int NCH, int HPW>
static cudaError_t run_decode_split(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  constexpr int D = NCH * 256;
  const size_t smem = sizeof(float) * (static_cast<size_t>(la.G) * D + 2 * kDecodeWarps * HPW +
                                       static_cast<size_t>(kDecodeWarps) * HPW * D);
  auto kern = decode_split_kernel<NCH, HPW>;
  // the shared-memory opt-in is per device and per size: set it when a call
  // needs more than this device was last given (never on every call)
  constexpr int kMaxDev = 64;
  static size_t attr_smem[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  if (smem > attr_smem[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    attr_smem[dev] = smem;
  }
  dim3 grid(da.nsplit, la.Hkv, da.B);
  kern<<<grid, kDecodeWarps * 32, smem, s>>>(da, la);
  return cudaGetLastError();
}

cudaError_t launch_decode_split(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  // bf16 or int8 caches: the tensor-core kernel (K=V, 8 or 16 query heads per kv head),
  // the persistent CUDA-core kernel (1, 2 or 4), else the split kernel below
  if (decode_tc_supported(la)) return launch_decode_tc(da, la, s);
  if (decode_simt_supported(la)) return launch_decode_simt(da, la, s);
  const int hpw = la.G <= 2 ? la.G : la.G / 4;
  if (la.D == 256) {
    switch (hpw) {
      case 1: return run_decode_split<1, 1>(da, la, s);
      case 2: return run_decode_split<1, 2>(da, la, s);
      case 4: return run_decode_split<1, 4>(da, la, s);
    }
  } else {
    switch (hpw) {
      case 1: return run_decode_split<2, 1>(da, la, s);
      case 2: return run_decode_split<2, 2>(da, la, s);
      case 4: return run_decode_split<2, 4>(da, la, s);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_decode_combine(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  const size_t smem = (static_cast<size_t>(da.nsplit) + 8) * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  if (la.D == 256) return launch_pdl(decode_combine_kernel<256>, dim3(la.H, da.B), dim3(128), smem, s, da, la);
  return launch_pdl(decode_combine_kernel<512>, dim3(la.H, da.B), dim3(128), smem, s, da, la);
}

// ---------------------------------------------------------------------------
// Self-test of the bounded wait: nothing ever arrives on the barrier.
// ---------------------------------------------------------------------------
__global__ void selftest_wait_kernel(uint32_t* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, timeout_ns, status, &abort_flag);
  __syncthreads();
}

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t timeout_ns, cudaStream_t s) {
  selftest_wait_kernel<<<1, 32, 0, s>>>(status, timeout_ns);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Workspace-free decode.  Its split partials live in this file-scope device
// array instead of a caller workspace; every GPU that loads the library keeps
// the array until the process exits.
// ---------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device.  In host code the array's name is only a host-side handle.
cudaError_t noalloc_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return cudaSuccess;
}

size_t round256(size_t x) { return (x + 255) / 256 * 256; }
}  // namespace

}  // namespace gattn

extern "C" int gattn_decode_noalloc(const gattn_bf16* q, const gattn_bf16* k_cache,
                                    const gattn_bf16* v_cache_or_null, const int32_t* seq_lens,
                                    gattn_bf16* out, int32_t batch, int32_t max_len,
                                    const gattn_cfg* cfg, gattn_stream stream) {
  using namespace gattn;
  LayerArgs la;
  int st = check_decode_call(cfg, q, k_cache, v_cache_or_null, seq_lens, out, batch, max_len, &la);
  if (st != GATTN_OK) return st;
  if (batch == 0) return GATTN_OK;

  // the normal split plan, with fewer (longer) splits when its partials
  // would not fit the scratch array
  DecodeArgs da;
  const size_t per_split = static_cast<size_t>(batch) * la.H * (la.D + 2) * sizeof(float);
  const size_t usable = kNoAllocScratchBytes - 512;  // room for two 256-byte roundings
  const size_t fit = usable / per_split;
  const int max_split = fit > (1u << 30) ? (1 << 30) : static_cast<int>(fit);
  if (max_split >= 1) decode_plan(la, batch, max_len, &da.nsplit, &da.chunk, max_split);
  if (max_split < 1 || da.nsplit > max_split) {
    // the layer's smallest plan still needs more split slots than fit: one
    // slot per chunk, and on the CUDA-core kernel's layers a chunk takes one
    // slot per warp-row group (8 / num_kv_heads of them)
    char msg[256];
    std::snprintf(msg, sizeof(msg),
                  "the smallest split plan of this layer needs %d slots of batch * num_heads * (head_dim + 2) * "
                  "4 = %zu bytes, more than the 16 MiB scratch of gattn_decode_noalloc holds (%d); use "
                  "gattn_decode with a workspace",
                  max_split < 1 ? 1 : da.nsplit, per_split, max_split < 0 ? 0 : max_split);
    return report_error(GATTN_ERR_UNSUPPORTED, msg);
  }
  void* base = nullptr;
  cudaError_t e = noalloc_scratch_address(&base);
  if (e != cudaSuccess) return report_error(GATTN_ERR_CUDA, "cudaGetSymbolAddress of the decode scratch failed");
  const size_t rows = static_cast<size_t>(batch) * la.H * da.nsplit;
  da.part_o = static_cast<float*>(base);
  da.part_ml = reinterpret_cast<float*>(static_cast<unsigned char*>(base) + round256(rows * la.D * sizeof(float)));
  da.q = reinterpret_cast<const __nv_bfloat16*>(q);
  da.k = reinterpret_cast<const __nv_bfloat16*>(k_cache);
  da.v = la.k_eq_v ? da.k : reinterpret_cast<const __nv_bfloat16*>(v_cache_or_null);
  da.seq_lens = seq_lens;
  da.out = reinterpret_cast<__nv_bfloat16*>(out);
  da.B = batch;
  da.max_len = max_len;
  da.status = nullptr;  // no status word: there is no workspace to hold one
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  e = launch_decode_split(da, la, s);
  if (e == cudaSuccess) e = launch_decode_combine(da, la, s);
  if (e != cudaSuccess) return report_error(GATTN_ERR_CUDA, cudaGetErrorString(e));
  return GATTN_OK;
}
