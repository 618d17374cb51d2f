// Split-KV decode on the tensor cores, for query groups of 8 or 16 heads per
// key/value head (the Gemma 4 global layer: 16 query heads on one K=V head).
//
// One CTA takes one chunk of one sequence's cache for one key/value head, in
// 128-key tiles.  With the keys as the MMA's M dimension ("swap AB"):
//   S^T [128 keys x 16] = K~ [128 x D] . Q~^T [D x 16]       (M=128, N=16)
//   O^T [D x 16]       += V^T [D x 128] . P^T [128 x 16]     (M=128 per 128 dims)
// (the group's G heads are the first G of the 16 columns).  A small
// tcgen05.mma costs a fixed ~46-77 cycles whatever N is, so 128 keys per
// instruction halve the Q K^T instruction count of 64-key tiles; a 128-key tile
// of head_dim 512 is 128 KB, too large to keep two of in shared memory for
// both products, so every tile streams through the shared-memory ring twice:
// once for Q K^T, its rotated dims rotated in place, and once more (from L2,
// where the first pass left it) for P V, as raw values.  The ring holds three
// 64 KB units (four 64-dim boxes of 128 keys); the producer streams Q K^T(j)
// units, then P V(j-1) units, so tile j's products overlap tile j-1's softmax.
// K~ is the raw key times the QK-norm gain, rotated, on dims [0, R); on the
// other dims the gain is folded into the query, and the key norm 1/rms(k) is a
// per-key scale of S^T.  With K=V the values are the raw tile.  The result is
// the same (m, l, O) partial per (b, head, chunk) as the other split kernels,
// merged by decode_combine_kernel.
//
// An int8 cache (Q8: codes c and one fp32 scale s per row, k = c * s) runs
// the same products on the codes themselves: integers in [-127, 127] are
// exact in fp16, which that instance's MMAs take (Q and P in fp16 as well).
// Each unit's codes land in the upper half of its slot, and the key warps
// widen them in place to the fp16 layout of the tile; the row
// scale then goes into the key's factor on S^T (s / sqrt(s^2 mean(c^2) + eps)
// under QK-norm, s without) and into P^T for P V (P(key) * s(key)), the
// softmax sums staying those of the unscaled P.
//
// Warps: 0-3 softmax over each tile's S^T (thread = key; TMEM lane = key) and
// the epilogue (thread = value dim); 4-11 two threads per key: int8 widening,
// key norms, the in-place rotation, and zeroing of rows past the chunk's end
// (so that P V multiplies 0 by 0 there, not by stale or poisoned data); 12 TMA
// producer; 13 MMA issuer.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "gattn_internal.h"
#include "kernels/common.cuh"
#include "kernels/rowops.cuh"

namespace gattn {

namespace {

template <int D, int G>
struct DecShape {
  static constexpr int TK = 128;                 // keys per tile
  static constexpr int BOX = TK * 128;           // 64 dims x 128 keys
  static constexpr int NBX = D / 64;             // boxes per tile
  static constexpr int UB = 4;                   // boxes per ring unit
  static constexpr int UNIT = UB * BOX;          // 64 KB
  static constexpr int NCH = NBX / UB;           // units per pass over a tile
  static constexpr int NSLOT = 3;                // ring units
  static constexpr int NQ = 16;                  // N of both products (G padded)
  static constexpr int QSLAB = NQ * 128;         // Q^T operand: 16 head rows x 64 dims
  static constexpr int PATOM = NQ * 128;         // P^T: 16 head rows x 64 keys
  static constexpr int PSLAB = 2 * PATOM;        // P^T of a 128-key tile
  static constexpr int OFF_RING = 0;
  static constexpr int OFF_Q = OFF_RING + NSLOT * UNIT;
  static constexpr int OFF_P = OFF_Q + NBX * QSLAB;
  static constexpr int OFF_RSTEP = OFF_P + 2 * PSLAB;        // (cos, sin) of a 128-position step, [64]
  static constexpr int OFF_RN = OFF_RSTEP + 64 * 8;          // key factor on S^T (1/rms, with int8 s/rms), [2][128]
  static constexpr int OFF_SC = OFF_RN + 2 * TK * 4;         // int8 row scales, [2][128]
  static constexpr int OFF_RED = OFF_SC + 2 * TK * 4;        // head maxima [2][4][16], sums [4][16]
  static constexpr int OFF_BAR = OFF_RED + 3 * 4 * 16 * 4;
  static constexpr int NBAR = 24;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TM_S0 = 0;           // S^T slots: 16 columns each
  static constexpr uint32_t TM_S1 = 16;
  static constexpr uint32_t TM_O = 32;           // O^T: D/128 blocks of 16 columns
  static constexpr uint32_t TMEM_COLS = 128;
  static constexpr int THREADS = 14 * 32;
  static_assert(G == 8 || G == 16, "query group of 8 or 16 heads");
  static_assert(NBX % UB == 0, "whole units");
  static_assert(TM_O + (D / 128) * NQ <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

// An int8 unit: its codes (two boxes of 128 dims x 128 keys) land in the upper
// half of the slot, then are widened to the four bf16 boxes in place.
constexpr int kQ8Box = 128 * 128;

struct DecTcParams {
  CUtensorMap tm_k;   // cache [B][Lmax][Hkv][D], box 64 dims x 128 keys (keys = values);
                      // int8 codes: box 128 dims x 128 keys
  DecodeArgs da;
  LayerArgs la;
  uint64_t timeout_ns;
};

constexpr float kLog2eD = 1.4426950408889634f;

// The MMA operands' element type: bf16 over a bf16 cache; fp16 over an int8
// cache (H), whose codes widen to fp16 in two operations per pair (below), Q
// and P then fp16 too (a kind::f16 MMA takes one type for A and B).
template <bool H>
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  if constexpr (H) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
  } else {
    return pack_bf16x2(lo, hi);
  }
}
template <bool H>
__device__ __forceinline__ void unpack8x(const uint4 u, float (&x)[8]) {
  if constexpr (H) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
      x[2 * e] = f.x;
      x[2 * e + 1] = f.y;
    }
  } else {
    unpack8(u, x);
  }
}
template <bool H>
__device__ __forceinline__ uint4 pack8x(const float (&x)[8]) {
  return make_uint4(pack2<H>(x[0], x[1]), pack2<H>(x[2], x[3]), pack2<H>(x[4], x[5]), pack2<H>(x[6], x[7]));
}
// Instruction descriptor of kind::f16 with fp16 A and B (the format fields of
// the bf16 descriptor cleared), fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return idesc_bf16_f32(M, N, a_mn_major, b_mn_major) & ~((7u << 7) | (7u << 10));
}

// Ring unit u of a chunk of n tiles: unit blocks in the order Q K^T(0),
// Q K^T(1), P V(0), Q K^T(2), P V(1), ..., Q K^T(n-1), P V(n-2), P V(n-1),
// each NCH units long.
struct UnitOf {
  int tile;
  bool pv;
  int c;    // unit within the pass
  int db;   // 256-dim block it holds (the rotated dims are in block 0, first)
};
template <int NCH>
__device__ __forceinline__ UnitOf unit_of(int u, int n) {
  const int blk = u / NCH;
  UnitOf r;
  r.c = u % NCH;
  if (blk == 0) {
    r.tile = 0;
    r.pv = false;
  } else if (blk == 2 * n - 1) {
    r.tile = n - 1;
    r.pv = true;
  } else if (blk & 1) {
    r.tile = (blk + 1) >> 1;
    r.pv = false;
  } else {
    r.tile = (blk >> 1) - 1;
    r.pv = true;
  }
  r.db = r.c;
  return r;
}

}  // namespace

template <int D, int G, bool Q8>
__global__ void __launch_bounds__(DecShape<D, G>::THREADS, 1) decode_tc_kernel(const __grid_constant__ DecTcParams P) {
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
  const int nunits = 2 * ntiles * C::NCH;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;            // [3] ring unit landed (TMA bytes)
  uint64_t* ready = bars + 3;       // [3] unit prepared by warps 4-11 (256 arrivals)
  uint64_t* empty = bars + 6;       // [3] the MMAs are done with the unit
  uint64_t* s_full = bars + 9;      // [2] S^T of a tile ready
  uint64_t* p_full = bars + 11;     // [2] P^T written, O rescaled, S read (128 arrivals)
  uint64_t* p_empty = bars + 13;    // [2] P V done with a P^T slot
  uint64_t* rn_full = bars + 15;    // [2] key norms of a tile written (256 arrivals)
  uint64_t* rn_empty = bars + 17;   // [2] the softmax has read them (128 arrivals)
  uint64_t* o_done = bars + 19;     // one phase per tile's P V
  uint64_t* o_final = bars + 20;
  uint64_t* q_ready = bars + 21;    // 256 arrivals (warps 0-7)
  uint64_t* drain = bars + 22;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  float* red = reinterpret_cast<float*>(smem + C::OFF_RED);    // [3][4][16]
  float* rnbuf = reinterpret_cast<float*>(smem + C::OFF_RN);   // [2][128]
  float* scbuf = reinterpret_cast<float*>(smem + C::OFF_SC);   // [2][128]
  const bool key_factor = Q8 || la.qk_norm;                     // a per-key factor on S^T

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSLOT; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&ready[i], 256);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&p_empty[i], 1);
      mbar_init(&rn_full[i], 256);
      mbar_init(&rn_empty[i], 128);
    }
    mbar_init(o_done, 1);
    mbar_init(o_final, 1);
    mbar_init(q_ready, 256);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 12 && lane == 0) tma_prefetch_desc(&P.tm_k);
  if (warp == 13) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = P.timeout_ns;

  if (warp < 8) {
    // ------------------------------------------------------------ query rows
    // Warps 0-7, one head per warp at a time: QK-norm and RoPE at position L-1
    // into the Q^T operand.  On the unrotated dims the key's gain is applied
    // here instead of to the keys.  Rows G..15 of Q^T and P^T stay zero.
    constexpr int NCHQ = D / 256;
    constexpr int HPW = (G + 7) / 8;
    const float koff = la.qk_norm == 1 ? 1.f : 0.f;
    const float4* gk4 = reinterpret_cast<const float4*>(la.k_norm_w);
    float x[HPW][NCHQ][8];
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) load_row<NCHQ>(da.q + (head0 + warp + 8 * hh) * D, lane, x[hh]);
#pragma unroll
    for (int hh = 0; hh < HPW; ++hh) {
      const int h = warp + 8 * hh;
      transform_row<NCHQ>(x[hh], lane, L - 1, la, la.q_norm_w, da.status);
#pragma unroll
      for (int i = 0; i < NCHQ; ++i) {
        const int c = lane + 32 * i;  // 8-dim chunk
        if (la.qk_norm && 8 * c >= la.rot) {
          const float4 g0 = __ldg(gk4 + 2 * c), g1 = __ldg(gk4 + 2 * c + 1);
          x[hh][i][0] *= g0.x + koff; x[hh][i][1] *= g0.y + koff;
          x[hh][i][2] *= g0.z + koff; x[hh][i][3] *= g0.w + koff;
          x[hh][i][4] *= g1.x + koff; x[hh][i][5] *= g1.y + koff;
          x[hh][i][6] *= g1.z + koff; x[hh][i][7] *= g1.w + koff;
        }
        *reinterpret_cast<uint4*>(smem + C::OFF_Q + (c >> 3) * C::QSLAB + h * 128 +
                                  (((c & 7) ^ (h & 7)) << 4)) = pack8x<Q8>(x[hh][i]);
      }
    }
    if constexpr (G < C::NQ) {
      // zero rows G..15 of every Q^T slab and of both P^T slots
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      for (int i = threadIdx.x; i < C::NBX * (C::NQ - G) * 8; i += 256) {
        const int sl = i / ((C::NQ - G) * 8), r = i % ((C::NQ - G) * 8);
        *reinterpret_cast<uint4*>(smem + C::OFF_Q + sl * C::QSLAB + G * 128 + r * 16) = z;
      }
      for (int i = threadIdx.x; i < 4 * (C::NQ - G) * 8; i += 256) {
        const int at = i / ((C::NQ - G) * 8), r = i % ((C::NQ - G) * 8);
        *reinterpret_cast<uint4*>(smem + C::OFF_P + at * C::PATOM + G * 128 + r * 16) = z;
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(q_ready);
  }
  if (warp < 4) {
    // ------------------------------------------------------------ softmax
    // Thread t serves key t of each tile: TMEM lane t holds its row of S^T with
    // the logits of all heads.  Maxima are per head over the tile's 128 keys
    // (warp shuffles, then the 4 warps through shared memory); the running max
    // m is the same in every thread, so the rescale decision is uniform.
    const int t = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const bool cap = la.softcap > 0.f;
    const float sl2 = la.scale_log2;
    const float kcap = cap ? la.scale / la.softcap : 0.f;
    const float cap_l2 = cap ? la.softcap * kLog2eD : 0.f;
    const bool odd = lane & 1;
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
      bool okj = ok && __all_sync(0xffffffffu, mbar_wait(&s_full[slot], par, tmo, da.status, abort_flag));
      float rn = 1.f, sk = 1.f;
      if (key_factor) {
        okj = okj && __all_sync(0xffffffffu, mbar_wait(&rn_full[slot], par, tmo, da.status, abort_flag));
        rn = rnbuf[slot * C::TK + t];
        if (Q8) sk = scbuf[slot * C::TK + t];
        mbar_arrive(&rn_empty[slot]);
      }
      float x[G];
      if (okj) {
        tc_fence_after();
        uint32_t sr[C::NQ];
        tmem_ldg<C::NQ>(tmem + lane_off + (slot ? C::TM_S1 : C::TM_S0), sr);
        tmem_wait_ld();
        const bool vis = (start + j * C::TK + t) < end;
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
        float* rw = red + (slot * 4 + warp) * 16;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float v = x[h];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == 0) rw[h] = v;
        }
        ok = named_barrier_and(1, 128, okj);
        if (!ok) break;
        const float* rr = red + slot * 4 * 16;
#pragma unroll
        for (int h = 0; h < G; ++h) {
          const float mt = fmaxf(fmaxf(rr[h], rr[16 + h]), fmaxf(rr[32 + h], rr[48 + h]));
          const float mn = fmaxf(m[h], mt);
          if (mn > m[h] + 8.f) {
            alpha[h] = m[h] == -INFINITY ? 0.f : ex2(m[h] - mn);
            any = any || m[h] != -INFINITY;
            m[h] = mn;
          }
        }
      }
      // P^T slot reuse: P V(j-2), which read it, must be complete
      if (!__all_sync(0xffffffffu, mbar_wait(&p_empty[slot], par ^ 1, tmo, da.status, abort_flag))) ok = false;
      // P^T row h: keys in two 64-key atoms, key k of an atom at 16-byte chunk
      // (k/8) ^ (h%8), half-word k%8.  Lanes 2i and 2i+1 (adjacent keys) swap
      // one value so that each writes a 32-bit word: the even lane for even
      // heads, the odd lane for odd heads.
      {
        uint8_t* pbase = smem + C::OFF_P + slot * C::PSLAB + (t >> 6) * C::PATOM;
        const int kp = t & 62;  // even key of the pair, within the atom
#pragma unroll
        for (int h = 0; h < G; h += 2) {
          float p0 = ex2(x[h] - (m[h] == -INFINITY ? 0.f : m[h]));
          float p1 = ex2(x[h + 1] - (m[h + 1] == -INFINITY ? 0.f : m[h + 1]));
          lp[h] = lp[h] * alpha[h] + p0;
          lp[h + 1] = lp[h + 1] * alpha[h + 1] + p1;
          if (Q8) {
            // P V runs on the codes: the key's scale goes into its P
            p0 *= sk;
            p1 *= sk;
          }
          const float recv = __shfl_xor_sync(0xffffffffu, odd ? p0 : p1, 1);
          const int hh = h + (odd ? 1 : 0);
          *reinterpret_cast<uint32_t*>(pbase + hh * 128 + (((kp >> 3) ^ (hh & 7)) << 4) + (kp & 7) * 2) =
              odd ? pack2<Q8>(recv, p1) : pack2<Q8>(p0, recv);
        }
      }
      // O must hold P V of every earlier tile before it is rescaled; seeing
      // S(j) implies P V(j-2) is complete, so o_done is at most one phase behind
      if (any && j >= 1) {
        const bool okw = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, tmo, da.status, abort_flag));
        if (okw) {
          tc_fence_after();
#pragma unroll
          for (int c = 0; c < D / 128; ++c) {
            uint32_t o[C::NQ];
            tmem_ldg<C::NQ>(tmem + lane_off + C::TM_O + c * C::NQ, o);
            tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < G; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * alpha[h]);
            tmem_stg<C::NQ>(tmem + lane_off + C::TM_O + c * C::NQ, o);
          }
          tmem_wait_st();
        } else {
          ok = false;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[slot]);
    }
    // Epilogue: l summed over the tile's keys and the 4 warps; thread t writes
    // value dim 128 c + t of each head's unnormalised O, lane t < G the (m, l)
    // of head t, in the split kernel's partial format.
    float* rl = red + 2 * 4 * 16;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float v = lp[h];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) rl[warp * 16 + h] = v;
    }
    ok = ok && __all_sync(0xffffffffu, mbar_wait(o_final, 0, tmo, da.status, abort_flag));
    ok = named_barrier_and(1, 128, ok);
    if (ok) {
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < D / 128; ++c) {
        uint32_t o[C::NQ];
        tmem_ldg<C::NQ>(tmem + lane_off + C::TM_O + c * C::NQ, o);
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
        ml[1] = ok ? (rl[h] + rl[16 + h]) + (rl[32 + h] + rl[48 + h]) : 0.f;
      }
    }
  }
  else if (warp < 12) {
    // ------------------------------------------------------- key preparation
    // Two threads per key (t8 = 2 k + hf) prepare each ring unit before the
    // MMAs read it.  Q K^T units: the key's sum of squares (QK-norm) over the
    // 16-byte chunks of its parity, and, in the first unit of a tile, the
    // rotated dims [0, R) of k * gain rotated in place.  P V units of a tile
    // that ends inside the chunk: rows past the end zeroed.  (cos, sin) of the
    // thread's pairs at its key's position: computed exactly (pair t turns
    // theta^(-2t/F) / 2pi per position, a geometric sequence in double
    // precision, reduced mod 1) every 32 tiles, and in between advanced by the
    // 128-position step of each pair.
    const int t8 = threadIdx.x - 128;
    const int k = t8 >> 1, hf = t8 & 1;
    const int R = la.rot;
    const int h8 = R >> 4;  // 8-dim chunks in half the rotated slice (<= 8)
    const float koff = la.qk_norm == 1 ? 1.f : 0.f;
    const float4* gk4 = reinterpret_cast<const float4*>(la.k_norm_w);
    float2* rstep = reinterpret_cast<float2*>(smem + C::OFF_RSTEP);
    constexpr double kTurnsPerRad = 0.15915494309189533576888376337251;
    if (t8 < (R >> 1)) {
      double f = kTurnsPerRad;
      for (int i = 0; i < t8; ++i) f *= la.rope_ratio;
      rstep[t8] = rope_cos_sin(C::TK, f);
    }
    named_barrier(2, 256);
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
    float ss = 0.f;
    // int8: the row scale of this thread's key in the current tile and the next
    float s_cur = 0.f, s_next = 0.f;
    auto load_scale = [&](int tile) -> float {
      const int key = start + tile * C::TK + k;
      return key < end ? __ldg(da.ks + (static_cast<size_t>(b) * da.max_len + key) * la.Hkv + kvh) : 0.f;
    };
    // the 256 threads leave the loop together, at a unit's first barrier, or
    // not at all (a failed wait is carried to the next unit in `okc`)
    bool okc = true;
    for (int u = 0; u < nunits; ++u) {
      const UnitOf uo = unit_of<C::NCH>(u, ntiles);
      const int slot = u % C::NSLOT;
      bool okw = okc && __all_sync(0xffffffffu, mbar_wait(&full[slot], (u / C::NSLOT) & 1, tmo, da.status,
                                                          abort_flag));
      if (!named_barrier_and(2, 256, okw)) break;
      uint8_t* ub = smem + C::OFF_RING + slot * C::UNIT;
      const int key0 = start + uo.tile * C::TK;
      const int nvalid = min(C::TK, end - key0);
      bool arrived = false;  // this unit already announced ready
      if constexpr (Q8) {
        // Widen the unit's codes (the slot's upper half: code box 0 = the
        // unit's dims 0-127, box 1 = dims 128-255; 128 B per key, 128-byte
        // swizzle) to the four fp16 boxes.  Box 0 goes to fp16 boxes 0-1 (the
        // lower half); box 1 is read by every thread before any of it is
        // overwritten by fp16 boxes 2-3.  A code c widens exactly: the fp16 of
        // bits 0x6400 | (c + 128) is 1024 + c + 128 (fp16 steps by 1 in
        // [1024, 2048)), so one byte permute places two codes under that
        // exponent byte and one packed subtract of 1152 leaves c.
        const uint8_t* q8 = ub + C::UNIT / 2;
        const __half2 k1152 = __floats2half2_rn(1152.f, 1152.f);
        auto widen = [&](const uint4 w, int cb) {  // 16 codes -> fp16 chunks cb, cb + 1
          const uint32_t ws[4] = {w.x ^ 0x80808080u, w.y ^ 0x80808080u, w.z ^ 0x80808080u, w.w ^ 0x80808080u};
          uint32_t h[8];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            // codes 4q, 4q+1 and 4q+2, 4q+3 as (low, high) halves
            uint32_t lo = __byte_perm(ws[q], 0x64646464u, 0x4140), hi = __byte_perm(ws[q], 0x64646464u, 0x4342);
            __half2 vl = __hsub2(*reinterpret_cast<__half2*>(&lo), k1152);
            __half2 vh = __hsub2(*reinterpret_cast<__half2*>(&hi), k1152);
            h[2 * q] = *reinterpret_cast<uint32_t*>(&vl);
            h[2 * q + 1] = *reinterpret_cast<uint32_t*>(&vh);
          }
          *tile_chunk(ub, C::BOX, k, cb) = make_uint4(h[0], h[1], h[2], h[3]);
          *tile_chunk(ub, C::BOX, k, cb + 1) = make_uint4(h[4], h[5], h[6], h[7]);
        };
        uint4 w1[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          const int i = hf + 2 * m;  // 16-code chunk of the box
          const int off = k * 128 + ((i ^ (k & 7)) << 4);
          const uint4 w0 = *reinterpret_cast<const uint4*>(q8 + off);
          w1[m] = *reinterpret_cast<const uint4*>(q8 + kQ8Box + off);
          widen(w0, 2 * i);
        }
        named_barrier(2, 256);
#pragma unroll
        for (int m = 0; m < 4; ++m) widen(w1[m], 16 + 2 * (hf + 2 * m));
        named_barrier(2, 256);
        if (!uo.pv && uo.c == 0) {
          // this tile's row scales (loaded a tile ahead) and the next tile's
          if (uo.tile == 0) s_next = load_scale(0);
          s_cur = s_next;
          s_next = uo.tile + 1 < ntiles ? load_scale(uo.tile + 1) : 0.f;
        }
      }
      if (!uo.pv) {
        if (la.qk_norm) {
          float acc[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll 4
          for (int c = hf; c < 4 * 8; c += 2) {
            float xx[8];
            unpack8x<Q8>(*tile_chunk(ub, C::BOX, k, c), xx);
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float2 v = make_float2(xx[e], xx[e + 1]);
              const float2 r2 = __ffma2_rn(v, v, make_float2(acc[e], acc[e + 1]));
              acc[e] = r2.x;
              acc[e + 1] = r2.y;
            }
          }
          ss += ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
        }
        if (uo.db == 0 && R > 0) {
          if (la.qk_norm) named_barrier(2, 256);  // every raw value is read before any is rotated
          // the angles at this tile's positions: exact every 32 tiles, else
          // advanced (after the previous tile's rotation) by one step
          if ((uo.tile & 31) == 0) anchor(checked_pos(min(key0 + k, end - 1), la, da.status));
          // all four chunk pairs loaded first, then rotated, so that their
          // latencies overlap; pairs past the rotated slice are not stored
          // (their chunks are still inside the unit's first two boxes)
          uint4 ux[4], uy[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = hf + 2 * i;
            ux[i] = *tile_chunk(ub, C::BOX, k, c);
            uy[i] = *tile_chunk(ub, C::BOX, k, c + h8);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int c = hf + 2 * i;
            float x[8], y[8];
            unpack8x<Q8>(ux[i], x);
            unpack8x<Q8>(uy[i], y);
            gain8(c, x);
            gain8(c + h8, y);
            // two pairs per packed fp32x2 instruction
            uint32_t xo[4], yo[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float2 co = make_float2(cs[i][e].x, cs[i][e + 1].x);
              const float2 si = make_float2(cs[i][e].y, cs[i][e + 1].y);
              const float2 x2 = make_float2(x[e], x[e + 1]), y2 = make_float2(y[e], y[e + 1]);
              const float2 a = __ffma2_rn(x2, co, __fmul2_rn(y2, make_float2(-si.x, -si.y)));
              const float2 bb = __ffma2_rn(y2, co, __fmul2_rn(x2, si));
              xo[e >> 1] = pack2<Q8>(a.x, a.y);
              yo[e >> 1] = pack2<Q8>(bb.x, bb.y);
            }
            if (c < h8) {
              *tile_chunk(ub, C::BOX, k, c) = make_uint4(xo[0], xo[1], xo[2], xo[3]);
              *tile_chunk(ub, C::BOX, k, c + h8) = make_uint4(yo[0], yo[1], yo[2], yo[3]);
            }
          }
          // the unit is ready for its MMAs now; the angles of the next tile
          // are advanced after (nothing waits for them until then)
          fence_proxy_async_smem();
          mbar_arrive(&ready[slot]);
          arrived = true;
          if (((uo.tile + 1) & 31) != 0) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int c = min(hf + 2 * i, 7);
#pragma unroll
              for (int e = 0; e < 8; e += 2) {
                // (cos, sin) of two pairs advanced by their steps, packed
                const float4 st = *reinterpret_cast<const float4*>(rstep + 8 * c + e);
                const float2 co = make_float2(cs[i][e].x, cs[i][e + 1].x);
                const float2 si = make_float2(cs[i][e].y, cs[i][e + 1].y);
                const float2 sc = make_float2(st.x, st.z), ss2 = make_float2(st.y, st.w);
                const float2 nc = __ffma2_rn(co, sc, __fmul2_rn(si, make_float2(-ss2.x, -ss2.y)));
                const float2 ns = __ffma2_rn(si, sc, __fmul2_rn(co, ss2));
                cs[i][e] = make_float2(nc.x, ns.x);
                cs[i][e + 1] = make_float2(nc.y, ns.y);
              }
            }
          }
        }
        if (uo.c == C::NCH - 1 && key_factor) {
          // the key's factor on S^T, read by the softmax per tile: 1/rms(k)
          // from both threads' sums; with int8 codes k = c s, so the factor is
          // s / sqrt(s^2 mean(c^2) + eps), or s without QK-norm
          float f = s_cur;
          if (la.qk_norm) {
            ss += __shfl_xor_sync(0xffffffffu, ss, 1);
            const float ms = ss / static_cast<float>(D);
            f = Q8 ? s_cur * rsqrtf(s_cur * s_cur * ms + la.eps) : rsqrtf(ms + la.eps);
          }
          ss = 0.f;
          const int ts = uo.tile & 1;
          okc = __all_sync(0xffffffffu, mbar_wait(&rn_empty[ts], ((uo.tile >> 1) & 1) ^ 1, tmo, da.status,
                                                  abort_flag));
          if (okc && hf == 0) {
            rnbuf[ts * C::TK + k] = f;
            if (Q8) scbuf[ts * C::TK + k] = s_cur;
          }
          mbar_arrive(&rn_full[ts]);
        }
      } else if (k >= nvalid) {
        const uint4 z = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 4
        for (int c = hf; c < 4 * 8; c += 2) *tile_chunk(ub, C::BOX, k, c) = z;
      }
      if (!arrived) {
        fence_proxy_async_smem();
        mbar_arrive(&ready[slot]);
      }
    }
  }
  else if (warp == 12) {
    // ------------------------------------------------------------- producer
    // One thread streams the ring units in the MMA issuer's order: each unit
    // (four 64-dim boxes of the tile's 128 keys) under one barrier phase,
    // once the MMAs are done with what the slot held.
    if (lane == 0) {
      int issued = 0;
      for (int u = 0; u < nunits; ++u) {
        const UnitOf uo = unit_of<C::NCH>(u, ntiles);
        const int slot = u % C::NSLOT;
        if (!mbar_wait(&empty[slot], ((u / C::NSLOT) & 1) ^ 1, tmo, da.status, abort_flag)) break;
        uint8_t* ub = smem + C::OFF_RING + slot * C::UNIT;
        mbar_arrive_expect_tx(&full[slot], Q8 ? C::UNIT / 2 : C::UNIT);
        if constexpr (Q8) {
#pragma unroll
          for (int bx = 0; bx < 2; ++bx)
            tma_load_4d(ub + C::UNIT / 2 + bx * kQ8Box, &P.tm_k, &full[slot], uo.db * 256 + bx * 128, kvh,
                        start + uo.tile * C::TK, b);
        } else {
#pragma unroll
          for (int bx = 0; bx < C::UB; ++bx)
            tma_load_4d(ub + bx * C::BOX, &P.tm_k, &full[slot], (uo.db * C::UB + bx) * 64, kvh,
                        start + uo.tile * C::TK, b);
        }
        issued = u + 1;
      }
      // let every issued copy land before the CTA can exit
      for (int u = issued - C::NSLOT < 0 ? 0 : issued - C::NSLOT; u < issued; ++u)
        mbar_wait(&full[u % C::NSLOT], (u / C::NSLOT) & 1, tmo, da.status, nullptr);
    }
  }
  else {
    // ------------------------------------------------------------ MMA issuer
    // Q K^T units: S^T(j) += K~ box . Q~^T box (A = key box, K-major, M=128;
    // B = Q^T slab, K-major, N=16); the first unit of tile j waits until the
    // softmax is done with S(j-2), whose TMEM slot it rewrites.  P V units:
    // O^T += V^T . P^T (A = two value boxes, MN-major, M=128 dims; B = P^T,
    // K-major, N=16); the first unit of tile j waits for P^T(j).
    if (lane == 0) {
      constexpr uint32_t idesc_qk = Q8 ? idesc_f16_f32(128, C::NQ, false, false) : idesc_bf16_f32(128, C::NQ, false, false);
      constexpr uint32_t idesc_pv = Q8 ? idesc_f16_f32(128, C::NQ, true, false) : idesc_bf16_f32(128, C::NQ, true, false);
      bool ok = mbar_wait(q_ready, 0, tmo, da.status, abort_flag);
      for (int u = 0; u < nunits && ok; ++u) {
        const UnitOf uo = unit_of<C::NCH>(u, ntiles);
        const int slot = u % C::NSLOT;
        const int ts = uo.tile & 1;
        const uint32_t tpar = (uo.tile >> 1) & 1;
        if (uo.c == 0)
          ok = uo.pv ? mbar_wait(&p_full[ts], tpar, tmo, da.status, abort_flag)
                     : mbar_wait(&p_full[ts], tpar ^ 1, tmo, da.status, abort_flag);
        ok = ok && mbar_wait(&ready[slot], (u / C::NSLOT) & 1, tmo, da.status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        const uint32_t ub = sbase + C::OFF_RING + slot * C::UNIT;
        if (!uo.pv) {
          const uint32_t s_tm = tmem + (ts ? C::TM_S1 : C::TM_S0);
#pragma unroll
          for (int bx = 0; bx < C::UB; ++bx) {
            const uint32_t qb = sbase + C::OFF_Q + (uo.db * C::UB + bx) * C::QSLAB;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss(s_tm, smem_desc_sw128(ub + bx * C::BOX + kk * 32, 16, 1024),
                          smem_desc_sw128(qb + kk * 32, 16, 1024), idesc_qk,
                          (uo.c > 0 || bx > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[slot]);
          if (uo.c == C::NCH - 1) mma_commit(&s_full[ts]);
        } else {
          const uint32_t pb = sbase + C::OFF_P + ts * C::PSLAB;
#pragma unroll
          for (int mbl = 0; mbl < 2; ++mbl) {
            const int mb = 2 * uo.db + mbl;  // 128-dim block of O^T
#pragma unroll
            for (int kk = 0; kk < C::TK / 16; ++kk)
              mma_bf16_ss(tmem + C::TM_O + mb * C::NQ,
                          smem_desc_sw128(ub + 2 * mbl * C::BOX + kk * 16 * 128, C::BOX, 1024),
                          smem_desc_sw128(pb + (kk >> 2) * C::PATOM + (kk & 3) * 32, 16, 1024), idesc_pv,
                          (uo.tile > 0 || kk > 0) ? 1u : 0u);
          }
          mma_commit(&empty[slot]);
          if (uo.c == C::NCH - 1) {
            mma_commit(&p_empty[ts]);
            mma_commit(o_done);
          }
        }
      }
      // o_final completes once every product above has; the TMEM they write
      // stays allocated until then
      mma_commit(o_final);
      mma_commit(drain);
      mbar_wait(drain, 0, tmo, da.status, nullptr);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int D, int G, bool Q8>
static cudaError_t run_decode_tc(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  using C = DecShape<D, G>;
  DecTcParams P;
  const bool enc = Q8 ? encode_tmap_bshd_u8(&P.tm_k, da.kq, da.B, da.max_len, la.Hkv, D, 128, C::TK)
                      : encode_tmap_bshd(&P.tm_k, da.k, da.B, da.max_len, la.Hkv, D, C::TK);
  if (!enc) return cudaErrorInvalidValue;
  P.da = da;
  P.la = la;
  P.timeout_ns = wait_timeout_ns();
  auto kern = decode_tc_kernel<D, G, Q8>;
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  kern<<<dim3(da.nsplit, la.Hkv, da.B), C::THREADS, C::SMEM, s>>>(P);
  return cudaGetLastError();
}

// (The C ABI has already checked that every cache pointer is 16-byte aligned.)
bool decode_tc_supported(const LayerArgs& la) {
  return la.k_eq_v && (la.G == 8 || la.G == 16) && (la.D == 256 || la.D == 512) && la.rot <= 128;
}

cudaError_t launch_decode_tc(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  if (da.kq) {
    if (la.D == 512)
      return la.G == 16 ? run_decode_tc<512, 16, true>(da, la, s) : run_decode_tc<512, 8, true>(da, la, s);
    return la.G == 16 ? run_decode_tc<256, 16, true>(da, la, s) : run_decode_tc<256, 8, true>(da, la, s);
  }
  if (la.D == 512)
    return la.G == 16 ? run_decode_tc<512, 16, false>(da, la, s) : run_decode_tc<512, 8, false>(da, la, s);
  return la.G == 16 ? run_decode_tc<256, 16, false>(da, la, s) : run_decode_tc<256, 8, false>(da, la, s);
}

}  // namespace gattn
