// Split-KV decode on the tensor cores, for query groups of 8 or 16 heads per
// key/value head (the Gemma 4 global layer: 16 query heads on one K=V head).
//
// One CTA takes one chunk of one sequence's cache for one key/value head, in
// 64-key tiles.  With the keys as the MMA's M dimension ("swap AB"):
//   S^T [64 keys x G heads] = K~ [64 x D] . Q~^T [D x G]        (M=64, N=G)
//   O^T [D x G]            += V^T [D x 64] . P^T [64 x G]       (M=128 per 128 dims)
// K~ is the raw key tile except on the rotated dims [0, R): those are rotated
// (and given the QK-norm gain) by CUDA cores into a small side tile, and the
// per-key norm 1/rms(k) is applied to S^T as a scale.  On the unrotated dims the
// gain is folded into the query instead.  With K=V the values are the raw tile
// already in shared memory.  The result is the same (m, l, O) partial per
// (b, head, chunk) as the SIMT split kernel, merged by decode_combine_kernel.
//
// Warps: 0-3 softmax over each tile's S^T (thread = key; TMEM lanes 0-15 of each
// quadrant hold the 64 rows of an M=64 accumulator) and the epilogue (thread =
// value dim); 4-7 the key prologue of each tile; 8 TMA producer; 9 MMA issuer.
#include <cuda_bf16.h>

#include "gattn_internal.h"
#include "kernels/common.cuh"
#include "kernels/rowops.cuh"

namespace gattn {

namespace {

template <int D, int G>
struct DecShape {
  static constexpr int TK = 64;                  // keys per tile
  static constexpr int BOX = TK * 128;           // 64 dims x 64 keys
  static constexpr int NB = D / 64;              // boxes per raw tile
  static constexpr int RAW = NB * BOX;           // raw key tile
  static constexpr int NSTAGE = 2;
  static constexpr int ROT_MAX = 128;            // rotated dims handled by the side tile
  static constexpr int ROTB = ROT_MAX / 64;      // side-tile boxes
  static constexpr int QSLAB = G * 128;          // Q^T operand: G head rows x 64 dims
  static constexpr int NPV = G < 16 ? 16 : G;    // N of P V (M=128 needs N % 16 == 0)
  static constexpr int PSLAB = NPV * 128;        // P^T: NPV head rows x 64 keys
  static constexpr int OFF_RAW = 0;
  static constexpr int OFF_ROT = OFF_RAW + NSTAGE * RAW;
  static constexpr int OFF_Q = OFF_ROT + NSTAGE * ROTB * BOX;
  static constexpr int OFF_P = OFF_Q + NB * QSLAB;
  static constexpr int OFF_RSTEP = OFF_P + NSTAGE * PSLAB;  // (cos, sin) of a 64-position step, [64]
  static constexpr int OFF_RED = OFF_RSTEP + 64 * 8;        // head maxima [2][4][G], sums [4][G]
  static constexpr int OFF_BAR = OFF_RED + 3 * 4 * G * 4;
  static constexpr int NBAR = 16;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TM_S0 = 0;           // S^T slots: G columns each
  static constexpr uint32_t TM_S1 = 32;
  static constexpr uint32_t TM_O = 64;           // O^T: D/128 chunks of NPV columns
  static constexpr uint32_t TMEM_COLS = 128;
  static_assert(G == 8 || G == 16, "query group of 8 or 16 heads");
  static_assert(TM_O + (D / 128) * NPV <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct DecTcParams {
  CUtensorMap tm_k;   // cache [B][Lmax][Hkv][D], box 64 dims x 64 keys (keys = values)
  DecodeArgs da;
  LayerArgs la;
  uint64_t timeout_ns;
};

constexpr float kLog2eD = 1.4426950408889634f;

}  // namespace

template <int D, int G>
__global__ void __launch_bounds__(320, 1) decode_tc_kernel(const __grid_constant__ DecTcParams P) {
  using C = DecShape<D, G>;
  const DecodeArgs& da = P.da;
  const LayerArgs& la = P.la;
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const size_t head0 = static_cast<size_t>(b) * la.H + static_cast<size_t>(kvh) * G;
  const int L = __ldg(da.seq_lens + b);
  const int lo = (L >= 1 && la.window > 0) ? max(0, L - la.window) : 0;
  const int start = lo + split * da.chunk;
  const int end = min(L, start + da.chunk);
  if (L < 1 || L > da.max_len || start >= end) {
    if ((L < 1 || L > da.max_len) && threadIdx.x == 0 && split == 0 && kvh == 0)
      flag_status(da.status, kStatusBounds);
    for (int h = threadIdx.x; h < G; h += blockDim.x) {
      float* ml = da.part_ml + ((head0 + h) * da.nsplit + split) * 2;
      ml[0] = -INFINITY;
      ml[1] = 0.f;
    }
    return;
  }
  const int ntiles = (end - start + C::TK - 1) / C::TK;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;            // [2] raw tile landed (TMA bytes)
  uint64_t* raw_empty = bars + 2;   // [2] P V done with the raw tile and P^T slot
  uint64_t* rot_full = bars + 4;    // [2] key prologue done (128 arrivals)
  uint64_t* rot_empty = bars + 6;   // [2] Q K^T done with the side tile
  uint64_t* s_full = bars + 8;      // [2] S^T ready
  uint64_t* p_full = bars + 10;     // [2] P^T written, O rescaled, S read (128 arrivals)
  // bars + 12: unused
  uint64_t* o_final = bars + 13;
  uint64_t* q_ready = bars + 14;    // 256 arrivals (warps 0-7)
  uint64_t* drain = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);    // [3][4][G]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&raw_empty[i], 1);
      mbar_init(&rot_full[i], 128);
      mbar_init(&rot_empty[i], 1);
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(o_final, 1);
    mbar_init(q_ready, 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) tma_prefetch_desc(&P.tm_k);
  if (warp == 9) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = P.timeout_ns;
  // optional timeline of this CTA (512 entries; layout in the public header)
  const long long cta = (static_cast<long long>(b) * la.Hkv + kvh) * da.nsplit + split;
  unsigned long long* trace =
      (da.trace && cta < static_cast<long long>(da.trace_bytes / (512 * sizeof(unsigned long long))))
          ? da.trace + cta * 512 : nullptr;
  const uint64_t t_start = trace ? globaltimer_ns() : 0;
  auto mark = [&](int slot) {
    if (trace) trace[slot] = globaltimer_ns() - t_start;
  };
  if (trace && threadIdx.x == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    trace[0] = t_start;
    trace[1] = smid;
    trace[2] = ntiles;
  }
  if (warp < 8) {
    // ------------------------------------------------------------ query rows
    // Warps 0-7, one head per warp at a time: QK-norm and RoPE at position L-1
    // into the Q^T operand.  On the unrotated dims the key's gain is applied
    // here instead of to the keys.  Every row is loaded before any is
    // transformed, so the global reads overlap.
    constexpr int NCH = D / 256;
    constexpr int HPW = (G + 7) / 8;
    const float koff = la.qk_norm == 1 ? 1.f : 0.f;
    const float4* gk4 = reinterpret_cast<const float4*>(la.k_norm_w);
    float x[HPW][NCH][8];
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) load_row<NCH>(da.q + (head0 + warp + 8 * hh) * D, lane, x[hh]);
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) {
      const int h = warp + 8 * hh;
      transform_row<NCH>(x[hh], lane, L - 1, la, la.q_norm_w, da.status);
#pragma unroll
      for (int i = 0; i < NCH; ++i) {
        const int c = lane + 32 * i;  // 8-dim chunk
        if (la.qk_norm && 8 * c >= la.rot) {
          const float4 g0 = __ldg(gk4 + 2 * c), g1 = __ldg(gk4 + 2 * c + 1);
          x[hh][i][0] *= g0.x + koff; x[hh][i][1] *= g0.y + koff;
          x[hh][i][2] *= g0.z + koff; x[hh][i][3] *= g0.w + koff;
          x[hh][i][4] *= g1.x + koff; x[hh][i][5] *= g1.y + koff;
          x[hh][i][6] *= g1.z + koff; x[hh][i][7] *= g1.w + koff;
        }
        *reinterpret_cast<uint4*>(smem + C::OFF_Q + (c >> 3) * C::QSLAB + h * 128 +
                                  (((c & 7) ^ (h & 7)) << 4)) = pack8(x[hh][i]);
      }
    }
    // P^T rows past the group (N padding of P V) stay zero
    if constexpr (C::NPV > G) {
      for (int i = threadIdx.x; i < 2 * (C::NPV - G) * 8; i += 256) {
        const int sl = i / ((C::NPV - G) * 8), r = i % ((C::NPV - G) * 8);
        *reinterpret_cast<uint4*>(smem + C::OFF_P + sl * C::PSLAB + G * 128 + r * 16) =
            make_uint4(0u, 0u, 0u, 0u);
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(q_ready);
  }
  if (warp < 4) {
    // ------------------------------------------------------------ softmax
    // Thread (warp w, lane i) serves key kt = 16 w + i%16 of each tile: lanes
    // i and i+16 sum the squares of its two halves of dims (the key's norm,
    // taken while the rotation and Q K^T run), and lane i < 16 reads its row
    // of S^T (TMEM lane 32 w + i holds row 16 w + i of an M=64 accumulator)
    // with the logits of all G heads.  Maxima are per head over the 64 keys
    // (warp shuffles, then the 4 warps through shared memory); the running
    // max m is the same in every thread, so the rescale decision is uniform
    // over the warpgroup.
    const int t = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const bool cap = la.softcap > 0.f;
    const float sl2 = la.scale_log2;
    const float kcap = cap ? la.scale / la.softcap : 0.f;
    const float cap_l2 = cap ? la.softcap * kLog2eD : 0.f;
    const int kt = 16 * warp + (lane & 15);  // key within the tile
    const int half = lane >> 4;
    const bool key_lane = lane < 16;
    float m[G], lp[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
      lp[h] = 0.f;
    }
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      const int slot = j & 1;
      const uint32_t par = (j >> 1) & 1;
      bool okj = ok && __all_sync(0xffffffffu, mbar_wait(&full[slot], par, tmo, da.status, abort_flag));
      float rn = 1.f;
      if (la.qk_norm) {
        float acc[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] = 0.f;
        if (okj) {
          uint8_t* raw = smem + C::OFF_RAW + slot * C::RAW;
#pragma unroll 4
          for (int c = half * (D / 16); c < (half + 1) * (D / 16); ++c) {
            float xx[8];
            unpack8(*tile_chunk(raw, C::BOX, kt, c), xx);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[e] = fmaf(xx[e], xx[e], acc[e]);
          }
        }
        float ss = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        ss += __shfl_xor_sync(0xffffffffu, ss, 16);
        rn = rsqrtf(ss / static_cast<float>(D) + la.eps);
      }
      if (t == 0 && j < 24) mark(176 + j);
      okj = okj && __all_sync(0xffffffffu, mbar_wait(&s_full[slot], par, tmo, da.status, abort_flag));
      if (t == 0 && j < 24) mark(80 + j);
      float x[G];
      if (okj) {
        tc_fence_after();
        uint32_t sr[G];
        tmem_ldg<G>(tmem + lane_off + (slot ? C::TM_S1 : C::TM_S0), sr);
        tmem_wait_ld();
        const bool vis = key_lane && (start + j * C::TK + kt) < end;
        const float f = rn * (cap ? kcap : sl2);
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float v = __uint_as_float(sr[h]) * f;
          x[h] = vis ? (cap ? cap_l2 * tanh_fast(v) : v) : -INFINITY;
        }
      } else {
#pragma unroll
        for (int h = 0; h < G; ++h) x[h] = -INFINITY;
      }
      // The running max moves only when a logit passes it by more than 8
      // (log2 units, a factor 256): the warpgroup votes, and exchanges the
      // tile's maxima only then.  Every thread of the warpgroup leaves the
      // loop at the exchange or not at all.
      bool need = !okj;
#pragma unroll
      for (int h = 0; h < G; ++h) need = need || x[h] > m[h] + 8.f;
      float alpha[G];
#pragma unroll
      for (int h = 0; h < G; ++h) alpha[h] = 1.f;
      bool any = false;
      if (named_barrier_or(1, 128, need)) {
        float* rw = red + (slot * 4 + warp) * G;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float v = x[h];
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
          v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
          if (lane == 0) rw[h] = v;
        }
        ok = named_barrier_and(1, 128, okj);
        if (!ok) break;
        const float* rr = red + slot * 4 * G;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mt = fmaxf(fmaxf(rr[h], rr[G + h]), fmaxf(rr[2 * G + h], rr[3 * G + h]));
          const float mn = fmaxf(m[h], mt);
          if (mn > m[h] + 8.f) {
            alpha[h] = m[h] == -INFINITY ? 0.f : ex2(m[h] - mn);
            any = any || m[h] != -INFINITY;
            m[h] = mn;
          }
        }
      }
      if (t == 0 && j < 24) mark(200 + j);
      // P^T slot reuse: P V(j-2), which read it, must be complete
      if (j >= 2) {
        if (!__all_sync(0xffffffffu, mbar_wait(&raw_empty[slot], par ^ 1, tmo, da.status, abort_flag)))
          ok = false;
      }
      if (t == 0 && j < 24) mark(248 + j);
      // P^T row h is one 128-byte swizzled row: key k at chunk (k/8) ^ (h%8),
      // half-word k%8.  Lanes 2i and 2i+1 (adjacent keys) swap one value so
      // that each writes a 32-bit word: the even lane for even heads, the odd
      // lane for odd heads.
      {
        uint8_t* pbase = smem + C::OFF_P + slot * C::PSLAB;
        const int kp = kt & ~1;
        const bool odd = lane & 1;
#pragma unroll
        for (int h = 0; h < G; h += 2) {
          const float p0 = ex2(x[h] - (m[h] == -INFINITY ? 0.f : m[h]));
          const float p1 = ex2(x[h + 1] - (m[h + 1] == -INFINITY ? 0.f : m[h + 1]));
          lp[h] = lp[h] * alpha[h] + p0;
          lp[h + 1] = lp[h + 1] * alpha[h + 1] + p1;
          const float recv = __shfl_xor_sync(0xffffffffu, odd ? p0 : p1, 1);
          if (key_lane) {
            const int hh = h + (odd ? 1 : 0);
            *reinterpret_cast<uint32_t*>(pbase + hh * 128 + (((kp >> 3) ^ (hh & 7)) << 4) + (kp & 7) * 2) =
                odd ? pack_bf16x2(recv, p1) : pack_bf16x2(p0, recv);
          }
        }
      }
      if (t == 0 && j < 24) mark(224 + j);
      // O must hold P V of every earlier tile before it is rescaled
      if (any && j >= 1) {
        const bool okw = __all_sync(0xffffffffu, mbar_wait(&raw_empty[(j - 1) & 1], ((j - 1) >> 1) & 1, tmo,
                                                           da.status, abort_flag));
        if (okw) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 128; ++c) {
            uint32_t o[C::NPV];
            tmem_ldg<C::NPV>(tmem + lane_off + C::TM_O + c * C::NPV, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
            tmem_stg<C::NPV>(tmem + lane_off + C::TM_O + c * C::NPV, o);
          }
          tmem_wait_st();
        } else {
          ok = false;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[slot]);
      if (lane == 0 && j < 24) mark((t == 0 ? 104 : 368 + 24 * warp) + j);
    }
    // Epilogue: l summed over the tile's keys and the 4 warps; thread t writes
    // value dim 128 c + t of each head's unnormalised O, lane t < G the (m, l)
    // of head t, in the split kernel's partial format.
    float* rl = red + 2 * 4 * G;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = lp[h];
      v += __shfl_xor_sync(0xffffffffu, v, 16);
      v += __shfl_xor_sync(0xffffffffu, v, 8);
      v += __shfl_xor_sync(0xffffffffu, v, 4);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      if (lane == 0) rl[warp * G + h] = v;
    }
    ok = ok && __all_sync(0xffffffffu, mbar_wait(o_final, 0, tmo, da.status, abort_flag));
    ok = named_barrier_and(1, 128, ok);
    if (t == 0) mark(4);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 128; ++c) {
        uint32_t o[C::NPV];
        tmem_ldg<C::NPV>(tmem + lane_off + C::TM_O + c * C::NPV, o);
        tmem_wait_ld();
#pragma unroll
        for (int h = 0; h < G; ++h)
          da.part_o[((head0 + h) * da.nsplit + split) * D + 128 * c + t] = __uint_as_float(o[h]);
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (t == h) {
        float* ml = da.part_ml + ((head0 + h) * da.nsplit + split) * 2;
        ml[0] = ok ? m[h] : -INFINITY;
        ml[1] = ok ? (rl[h] + rl[G + h]) + (rl[2 * G + h] + rl[3 * G + h]) : 0.f;
      }
    }
  }
  else if (warp < 8) {
    // ------------------------------------------------------------ key prologue
    // Two threads per key (t4 = 2 k + hf) write the rotated dims [0, R) of
    // k * gain into the side tile, and zero rows for keys past the chunk's end
    // so that P V multiplies 0 by 0 there, not by stale data.  Each thread
    // keeps (cos, sin) of its pairs' angles at its key's position: computed
    // exactly (pair t turns theta^(-2t/F) / 2pi per position, a geometric
    // sequence in double precision, reduced mod 1) every 32 tiles, and in
    // between advanced by the 64-position step of each pair.
    const int t4 = threadIdx.x - 128;
    const int k = t4 >> 1, hf = t4 & 1;
    const int R = la.rot;
    const int h8 = R >> 4;                  // 8-dim chunks in half the rotated slice (<= 8)
    const int rch = ((R + 63) >> 6) << 3;   // chunks covered by the side tile's boxes
    const float koff = la.qk_norm == 1 ? 1.f : 0.f;
    const float4* gk4 = reinterpret_cast<const float4*>(la.k_norm_w);
    float2* rstep = reinterpret_cast<float2*>(smem + C::OFF_RSTEP);
    constexpr double kTurnsPerRad = 0.15915494309189533576888376337251;
    if (t4 < (R >> 1)) {
      double f = kTurnsPerRad;
      for (int i = 0; i < t4; ++i) f *= la.rope_ratio;
      rstep[t4] = rope_cos_sin(C::TK, f);
    }
    named_barrier(2, 128);
    float2 cs[4][8];
    auto anchor = [&](int pos) {
      double qp[8];
      qp[0] = 1.0;
#pragma unroll
      for (int e = 1; e < 8; ++e) qp[e] = qp[e - 1] * la.rope_ratio;
      const double q8 = qp[7] * la.rope_ratio;
      const double q16 = q8 * q8;
      double f8 = kTurnsPerRad * (hf ? q8 : 1.0);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (hf + 2 * i < h8) {
#pragma unroll
          for (int e = 0; e < 8; ++e) cs[i][e] = rope_cos_sin(pos, f8 * qp[e]);
        }
        f8 *= q16;
      }
    };
    auto gain8 = [&](int c, float (&x)[8]) {
      if (!la.qk_norm) return;
      const float4 g0 = __ldg(gk4 + 2 * c), g1 = __ldg(gk4 + 2 * c + 1);
      x[0] *= g0.x + koff; x[1] *= g0.y + koff; x[2] *= g0.z + koff; x[3] *= g0.w + koff;
      x[4] *= g1.x + koff; x[5] *= g1.y + koff; x[6] *= g1.z + koff; x[7] *= g1.w + koff;
    };
    for (int j = 0; j < ntiles; ++j) {
      const int slot = j & 1;
      const uint32_t par = (j >> 1) & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&full[slot], par, tmo, da.status, abort_flag) &&
                                       mbar_wait(&rot_empty[slot], par ^ 1, tmo, da.status, abort_flag)))
        break;
      if (t4 == 0 && j < 24) mark(8 + j);
      uint8_t* raw = smem + C::OFF_RAW + slot * C::RAW;
      uint8_t* rot = smem + C::OFF_ROT + slot * C::ROTB * C::BOX;
      const int key = start + j * C::TK + k;
      if (R > 0) {
        if ((j & 31) == 0) {
          anchor(checked_pos(min(key, end - 1), la, da.status));
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = hf + 2 * i;
            if (c < h8) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const float2 st = rstep[8 * c + e];
                const float2 a = cs[i][e];
                cs[i][e] = make_float2(a.x * st.x - a.y * st.y, a.y * st.x + a.x * st.y);
              }
            }
          }
        }
      }
      if (t4 == 0 && j < 24) mark(296 + j);
      if (key < end) {
        if (R > 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = hf + 2 * i;
            if (c < h8) {
              float x[8], y[8];
              unpack8(*tile_chunk(raw, C::BOX, k, c), x);
              unpack8(*tile_chunk(raw, C::BOX, k, c + h8), y);
              gain8(c, x);
              gain8(c + h8, y);
              float xo[8], yo[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                xo[e] = x[e] * cs[i][e].x - y[e] * cs[i][e].y;
                yo[e] = y[e] * cs[i][e].x + x[e] * cs[i][e].y;
              }
              *tile_chunk(rot, C::BOX, k, c) = pack8(xo);
              *tile_chunk(rot, C::BOX, k, c + h8) = pack8(yo);
            }
          }
          // unrotated dims that share a box with rotated ones: copied raw
          for (int c = 2 * h8 + hf; c < rch; c += 2) *tile_chunk(rot, C::BOX, k, c) = *tile_chunk(raw, C::BOX, k, c);
        }
      } else {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
        for (int c = hf; c < D / 8; c += 2) *tile_chunk(raw, C::BOX, k, c) = z;
        for (int c = hf; c < rch; c += 2) *tile_chunk(rot, C::BOX, k, c) = z;
      }
      fence_proxy_async_smem();
      mbar_arrive(&rot_full[slot]);
      if ((t4 & 31) == 0 && j < 24) mark((t4 == 0 ? 32 : 296 + t4 * 3 / 4) + j);
    }
  }
  else if (warp == 8) {
    // ------------------------------------------------- TMA producer, P V issuer
    // One thread loads tiles 0 and 1, then per tile j issues
    // O^T += V^T P^T once the softmax has written P^T(j): A = value boxes
    // (MN-major, M=128 dims over two 64-dim boxes LBO apart), B = P^T
    // (K-major, N=NPV); and once that P V has completed, loads tile j+2 into
    // the slot it frees.
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, C::NPV, true, false);
      // Tiles beyond the two shared-memory slots are brought into L2 ahead of
      // their loads (up to kPrefetch tiles past the one being loaded), so a
      // slot that frees up refills from L2 instead of waiting on HBM.
      constexpr int kPrefetch = 4;
      int pf_next = 2;
      auto load = [&](int j) {
        const int slot = j & 1;
        mbar_arrive_expect_tx(&full[slot], C::RAW);
#pragma unroll
        for (int c = 0; c < C::NB; ++c)
          tma_load_4d(smem + C::OFF_RAW + slot * C::RAW + c * C::BOX, &P.tm_k, &full[slot], 64 * c,
                      kvh, start + j * C::TK, b);
        for (; pf_next < ntiles && pf_next <= j + kPrefetch; ++pf_next)
#pragma unroll
          for (int c = 0; c < C::NB; ++c) tma_prefetch_l2_4d(&P.tm_k, 64 * c, kvh, start + pf_next * C::TK, b);
        if (j < 24) mark(152 + j);
      };
      int issued = 0;
      for (; issued < 2 && issued < ntiles; ++issued) load(issued);
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        const int slot = j & 1;
        const uint32_t par = (j >> 1) & 1;
        ok = mbar_wait(&p_full[slot], par, tmo, da.status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t rawb = sbase + C::OFF_RAW + slot * C::RAW;
        const uint32_t pb = sbase + C::OFF_P + slot * C::PSLAB;
#pragma unroll
        for (int mc = 0; mc < D / 128; ++mc)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(tmem + C::TM_O + mc * C::NPV,
                        smem_desc_sw128(rawb + 2 * mc * C::BOX + kk * 2048, C::BOX, 1024),
                        smem_desc_sw128(pb + kk * 32, 16, 1024), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&raw_empty[slot]);
        if (j < 24) mark(128 + j);
        if (j + 2 < ntiles) {
          ok = mbar_wait(&raw_empty[slot], par, tmo, da.status, abort_flag);
          if (!ok) break;
          load(j + 2);
          issued = j + 3;
        }
      }
      // o_final completes once every P V above has; the TMEM they write
      // stays allocated until then
      mma_commit(o_final);
      mbar_wait(o_final, 0, tmo, da.status, nullptr);
      // let every issued copy land before the CTA can exit
      for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j)
        mbar_wait(&full[j & 1], (j >> 1) & 1, tmo, da.status, nullptr);
    }
  }
  else {
    // ------------------------------------------------------------ MMA issuer
    // S^T = K~ Q~^T: A = key box (K-major, M=64; the side tile's boxes on the
    // rotated dims), B = Q^T slab (K-major, N=G).  Q K^T(j) waits for its
    // tile, its side tile, and for the softmax to be done with S(j-2), whose
    // TMEM slot it rewrites.
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(64, G, false, false);
      const int rotb = (la.rot + 63) >> 6;
      bool ok = mbar_wait(q_ready, 0, tmo, da.status, abort_flag);
      mark(3);
      // The unrotated dims go first, as soon as the tile has landed; the
      // rotated ones (from the side tile) once the key prologue is done.
      for (int j = 0; j < ntiles && ok; ++j) {
        const int slot = j & 1;
        const uint32_t par = (j >> 1) & 1;
        ok = mbar_wait(&full[slot], par, tmo, da.status, abort_flag) &&
             (j < 2 || mbar_wait(&p_full[slot], par ^ 1, tmo, da.status, abort_flag));
        if (!ok) break;
        tc_fence_after();
        const uint32_t s_tm = tmem + (slot ? C::TM_S1 : C::TM_S0);
        const uint32_t rawb = sbase + C::OFF_RAW + slot * C::RAW;
        const uint32_t rotbase = sbase + C::OFF_ROT + slot * C::ROTB * C::BOX;
        for (int c = rotb; c < C::NB; ++c) {
          const uint32_t ab = rawb + c * C::BOX;
          const uint32_t qb = sbase + C::OFF_Q + c * C::QSLAB;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(s_tm, smem_desc_sw128(ab + kk * 32, 16, 1024),
                        smem_desc_sw128(qb + kk * 32, 16, 1024), idesc_qk, (c > rotb || kk > 0) ? 1u : 0u);
        }
        if (j < 24) mark(56 + j);
        ok = mbar_wait(&rot_full[slot], par, tmo, da.status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        for (int c = 0; c < rotb; ++c) {
          const uint32_t ab = rotbase + c * C::BOX;
          const uint32_t qb = sbase + C::OFF_Q + c * C::QSLAB;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_bf16_ss(s_tm, smem_desc_sw128(ab + kk * 32, 16, 1024),
                        smem_desc_sw128(qb + kk * 32, 16, 1024), idesc_qk,
                        (rotb < C::NB || c > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&rot_empty[slot]);
        mma_commit(&s_full[slot]);
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, tmo, da.status, nullptr);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0) mark(5);
}

template <int D, int G>
static cudaError_t run_decode_tc(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  using C = DecShape<D, G>;
  DecTcParams P;
  if (!encode_tmap_bshd(&P.tm_k, da.k, da.B, da.max_len, la.Hkv, D, C::TK))
    return cudaErrorInvalidValue;
  P.da = da;
  P.la = la;
  P.timeout_ns = wait_timeout_ns();
  auto kern = decode_tc_kernel<D, G>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  kern<<<dim3(da.nsplit, la.Hkv, da.B), 320, C::SMEM, s>>>(P);
  return cudaGetLastError();
}

// (The C ABI has already checked that every cache pointer is 16-byte aligned.)
bool decode_tc_supported(const LayerArgs& la) {
  return la.k_eq_v && (la.G == 8 || la.G == 16) && (la.D == 256 || la.D == 512) && la.rot <= 128;
}

cudaError_t launch_decode_tc(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  if (la.D == 512) return la.G == 16 ? run_decode_tc<512, 16>(da, la, s) : run_decode_tc<512, 8>(da, la, s);
  return la.G == 16 ? run_decode_tc<256, 16>(da, la, s) : run_decode_tc<256, 8>(da, la, s);
}

}  // namespace gattn
