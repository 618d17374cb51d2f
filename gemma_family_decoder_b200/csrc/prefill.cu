// Prefill self-attention on the sm_100a tensor cores (tcgen05 + TMA + TMEM).
//
// A persistent kernel: one CTA per SM takes work items in turn, an item being
// a 128-query tile of one head (and, for head_dim 512, one 256-wide half of
// the value dims), heaviest items first.  The queries arrive already normed
// and rotated (the prologue kernel).  Warp roles:
//   warps 0-3  per KV tile: S from TMEM -> scale (and softcap) -> causal/window
//              mask on boundary tiles only -> online softmax with lazy rescale
//              -> P (bf16) written back into the same TMEM columns; at the
//              end of an item, O / l -> bf16 straight to global memory.
//   warp 4     TMA producer: per item the first key tile, the Q tile (once the
//              previous item's last Q K^T is done with the buffer), then key
//              and value tiles, each under one barrier phase, into a ring of
//              one key tile and one value tile.
//   warp 5     MMA issuer: S = Q K^T into a double-buffered TMEM slot, then
//              O += P V with P read from that slot, into the TMEM accumulator.
// Because P lives in the S slot, the softmax of tile j+1 never waits for the
// P V product of tile j (it waits only in the rare case that O must be
// rescaled), and the tensor core runs Q K^T of tile j+1 while the softmax of
// tile j is still being computed.  Barrier phases count tiles and items over
// the whole run of a CTA, so the next item's loads start while the current
// one finishes.  KV tiles entirely outside the causal window are never visited.
//
// Layer definition: KerasFormers "Gemma 4" (What changed: plain-weight RMSNorm,
// partial rotation, K=V global layers), KerasFormers "Gemma 3" (What changed:
// dual RoPE bases), ZeroModels "Gemma 2" (logit softcapping, alternating
// sliding-window attention, query_pre_attn_scalar).
#include <cuda_bf16.h>

#include "gattn_internal.h"
#include "kernels/common.cuh"
#include "kernels/rowops.cuh"

namespace gattn {

using bf16 = __nv_bfloat16;

template <int D, int BN>
struct PrefillShape {
  static constexpr int BM = 128;
  static constexpr int DV = 256;                 // value dims per CTA
  static constexpr int SLAB_KV = BN * 128;       // one 64-dim TMA box of BN rows = one slot
  static constexpr int KCH = D / 64;             // slots per key tile
  static constexpr int VCH = DV / 64;            // slots per value tile
  static constexpr int SLAB128 = BM * 128;       // 64 dims x 128 rows
  static constexpr int Q_BYTES = (D / 64) * SLAB128;
  // ring slots: a multiple of 4 so that every 4-slot value tile is contiguous
  static constexpr int NSTAGE = ((227 * 1024 - Q_BYTES - 2048) / SLAB_KV) / 4 * 4;
  static constexpr int OFF_RING = Q_BYTES;
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_BAR = OFF_RING + NSTAGE * SLAB_KV;
  static constexpr int NBAR = 2 * NSTAGE + 10;
  static_assert(NSTAGE >= KCH + VCH, "ring must hold a key tile and a value tile");
  static_assert(KCH % 4 == 0 && VCH == 4 && NSTAGE % 4 == 0, "value tiles must not wrap the ring");
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack to align the base to 1 KB
  static constexpr uint32_t TM_O = 0;
  static constexpr uint32_t TM_S0 = DV;
  static constexpr uint32_t TM_S1 = TM_S0 + BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(TM_S1 + BN <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(NSTAGE == KCH + VCH, "the ring is one key tile and one value tile");
};

struct PrefillKParams {
  CUtensorMap tm_q;
  CUtensorMap tm_k;
  CUtensorMap tm_v;
  __nv_bfloat16* out;
  uint32_t* status;
  uint64_t timeout_ns;
  int B, S, nqt, dv_splits;
  LayerArgs la;
  unsigned long long* trace;  // optional per-CTA event times (kTraceSlots each), or null
  int trace_ctas;
  const int* seq_range;       // [B][2] valid tokens [lo, hi) of each sequence, or null (all valid)
  const int* q_off;           // chunk: token index of each sequence's first query row
  int KV_S;                   // chunk: key/value rows (the cache length)
};

// Optional timeline of one CTA's first item (debug aid, off unless a trace
// buffer is set): [0] start time (ns), [1] SM id, [2] KV tiles, [3] Q landed
// at the MMA warp, [4] epilogue start, [5] end of the CTA, [6] first key tile
// landed, [7] items of the CTA, then per KV tile j (j < 120): [8+j] S(j) seen
// by the softmax, [128+j] P(j) written, [248+j] Q K^T(j) issued, [368+j]
// P V(j) issued; times relative to [0].
constexpr int kTraceSlots = 512;

constexpr float kLog2e = 1.4426950408889634f;

// MODE 0: a whole prompt; 1: a padded batch (P.seq_range); 2: a chunk of S
// queries against a cache of KV_S rows, query row i of sequence b being token
// q_off[b] + i.  Separate instances, so the plain kernel carries none of the
// extra index arithmetic.
template <int D, int BN, bool CAP, int MODE>
__global__ void __launch_bounds__(192, 1) prefill_kernel(const __grid_constant__ PrefillKParams P) {
  using C = PrefillShape<D, BN>;
  constexpr bool PAD = MODE == 1, CHUNK = MODE == 2;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* kf = bars;          // key tile landed (one phase per KV tile)
  uint64_t* ke = bars + 1;      // Q K^T done with the key tile
  uint64_t* vf = bars + 2;      // value tile landed
  uint64_t* ve = bars + 3;      // P V done with the value tile
  uint64_t* s_full = bars + 4;  // [2] S ready in its TMEM slot
  uint64_t* p_full = bars + 6;  // [2] P written over it (128 arrivals)
  uint64_t* o_done = bars + 8;  // one phase per P V
  uint64_t* q_full = bars + 9;  // Q tile landed (one phase per item)
  uint64_t* q_empty = bars + 10;  // the item's last Q K^T is done with the Q tile
  uint64_t* o_final = bars + 11;  // the item's last P V is done
  uint64_t* o_empty = bars + 12;  // the softmax has read the item's O (128 arrivals)
  uint64_t* drain = bars + 13;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const LayerArgs& la = P.la;
  const int H = la.H, S = P.S;
  const int nitems = P.nqt * P.B * H * P.dv_splits;
  // work item `it`, heaviest query tiles first
  struct Item {
    int qt, dvs, h, b, kvh, q0, dv_lo, k_first, ntiles, rot;
    int lo, hi;  // the sequence's valid tokens (all of [0, S) unless the batch is padded)
    int qa;      // token index of the tile's first row (q0 unless a chunk)
  };
  auto item_of = [&](int it) {
    Item w;
    const int per_qt = P.B * H * P.dv_splits;
    w.qt = P.nqt - 1 - it / per_qt;
    int idx = it % per_qt;
    w.dvs = idx % P.dv_splits;
    idx /= P.dv_splits;
    w.h = idx % H;
    w.b = idx / H;
    w.kvh = w.h / la.G;
    w.q0 = w.qt * C::BM;
    w.dv_lo = w.dvs * C::DV;
    w.lo = 0;
    w.hi = S;
    w.qa = w.q0;
    if constexpr (PAD) {
      w.lo = min(max(__ldg(P.seq_range + 2 * w.b), 0), S);
      w.hi = min(max(__ldg(P.seq_range + 2 * w.b + 1), 0), S);
    }
    if constexpr (CHUNK) {
      // the chunk's tokens [off, off + S) of a cache of KV_S rows
      const int off = min(max(__ldg(P.q_off + w.b), 0), P.KV_S - S);
      w.qa = w.q0 + off;
      w.hi = off + S;
    }
    // keys of the tile's valid rows: from the window's (and the sequence's)
    // first key to the last valid row
    const int kv_hi = min(min(CHUNK ? w.hi : S, w.qa + C::BM), w.hi);
    const int kv_lo = max(la.window > 0 ? max(0, w.qa - la.window + 1) : 0, w.lo);
    w.k_first = (kv_lo / BN) * BN;
    // a query tile with no valid row reads no keys: its rows are zero
    const bool none = PAD && (w.lo >= w.hi || w.q0 + C::BM <= w.lo || w.q0 >= w.hi);
    w.ntiles = none ? 0 : (kv_hi - w.k_first + BN - 1) / BN;
    // KV tiles are visited starting at a tile that differs between the items
    // working on one sequence at once, so they do not all read the same L2
    // lines together (the online softmax is independent of the visiting order)
    w.rot = w.ntiles > 1 ? (w.h * 7 + w.dvs * 3 + w.b * 5 + w.qt) % w.ntiles : 0;
    return w;
  };
  auto tile_key = [&](const Item& w, int j) { return w.k_first + ((j + w.rot) % w.ntiles) * BN; };
  // This CTA's items: round r gives it item r*G + c, or r*G + G-1-c on odd
  // rounds, so that the heaviest-first items spread evenly over the CTAs.
  const int G = gridDim.x, cta = blockIdx.x;
  const int nrounds = (nitems + G - 1) / G;
  auto item_at = [&](int r) { return r * G + ((r & 1) ? G - 1 - cta : cta); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
    }
    mbar_init(kf, 1);
    mbar_init(ke, 1);
    mbar_init(vf, 1);
    mbar_init(ve, 1);
    mbar_init(o_done, 1);
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(o_final, 1);
    mbar_init(o_empty, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&P.tm_q);
    tma_prefetch_desc(&P.tm_k);
    tma_prefetch_desc(&P.tm_v);
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // the prologue kernel's queries and keys are complete and visible past here
  pdl_wait();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = P.timeout_ns;
  unsigned long long* trace = (P.trace && static_cast<int>(blockIdx.x) < P.trace_ctas)
                                  ? P.trace + static_cast<size_t>(blockIdx.x) * kTraceSlots : nullptr;
  const uint64_t t_start = globaltimer_ns();
  auto mark = [&](int slot) {
    if (trace) trace[slot] = globaltimer_ns() - t_start;
  };
  if (trace && threadIdx.x == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    trace[0] = t_start;
    trace[1] = smid;
    int n = 0;
    for (int r = 0; r < nrounds; ++r) n += item_at(r) < nitems;
    trace[2] = item_of(item_at(0)).ntiles;
    trace[7] = n;
  }

  if (warp < 4) {
    // ------------------------------------------------------------------ softmax
    const int t = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = la.scale_log2;
    const float kcap = CAP ? la.scale / la.softcap : 0.f;
    const float cap_l2 = CAP ? la.softcap * kLog2e : 0.f;
    const int W = la.window;
    bool ok = true;
    int T0 = 0;  // KV tiles of this CTA's earlier items
    for (int r = 0, I = 0; r < nrounds && ok; ++r) {
      const int it = item_at(r);
      if (it >= nitems) continue;
      const Item w = item_of(it);
      const int qi = w.q0 + t;
      const bool in_seq = qi < S;                            // a row of the output
      const bool valid = in_seq && (!PAD || (qi >= w.lo && qi < w.hi));  // and not padding
      const int qa = w.qa + t;                               // its token index
      if (PAD && t == 0 && w.qt == 0 && w.h == 0 && w.dvs == 0) {
        const int lo_in = __ldg(P.seq_range + 2 * w.b), hi_in = __ldg(P.seq_range + 2 * w.b + 1);
        if (lo_in < 0 || hi_in > S) flag_status(P.status, kStatusBounds);
      }
      if (CHUNK && t == 0 && w.qt == 0 && w.h == 0 && w.dvs == 0) {
        const int off_in = __ldg(P.q_off + w.b);
        if (off_in < 0 || off_in > P.KV_S - S) flag_status(P.status, kStatusBounds);
      }
      if (PAD && w.ntiles == 0) {
        // every row of the tile is padding: zero output, no keys, no MMAs
        if (in_seq) {
          uint4* orow = reinterpret_cast<uint4*>(P.out + ((static_cast<size_t>(w.b) * S + qi) * H + w.h) * D + w.dv_lo);
          for (int c = 0; c < C::DV / 8; ++c) orow[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        continue;
      }
      float m = -INFINITY, l = 0.f;
      for (int j = 0; j < w.ntiles && ok; ++j) {
        const int T = T0 + j;
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[T & 1], (T >> 1) & 1, tmo, P.status, abort_flag));
        if (!ok) break;
        if (t == 0 && I == 0 && j < 120) mark(8 + j);
        tc_fence_after();
        const uint32_t scol = tmem + lane_off + ((T & 1) ? C::TM_S1 : C::TM_S0);
        uint32_t rr[BN / 32][32];
#pragma unroll
        for (int c = 0; c < BN / 32; ++c) tmem_ld32(scol + c * 32, rr[c]);
        tmem_wait_ld();

        const int key0 = tile_key(w, j);
        const bool full_tile = (key0 + BN - 1 <= w.qa) && (w.q0 + C::BM <= (PAD ? min(S, w.hi) : S)) &&
                               (!PAD || (key0 >= w.lo && w.q0 >= w.lo)) &&
                               (W <= 0 || (w.qa + C::BM - 1) - key0 < W);
        float x[BN];
#pragma unroll
        for (int i = 0; i < BN; ++i) {
          const float sv = __uint_as_float(rr[i >> 5][i & 31]);
          x[i] = CAP ? cap_l2 * tanh_fast(sv * kcap) : sv;
        }
        if (!full_tile) {
          const int hi = valid ? qa - key0 : -1;            // visible iff i <= hi
          const int lo_w = W > 0 ? qa - key0 - W + 1 : -BN;   // and i >= lo
          const int lo = PAD ? max(lo_w, w.lo - key0) : lo_w;
#pragma unroll
          for (int i = 0; i < BN; ++i) x[i] = (i <= hi && i >= lo) ? x[i] : -INFINITY;
        }
        float mxa[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) mxa[a] = x[a];
#pragma unroll
        for (int i = 8; i < BN; ++i) mxa[i & 7] = fmaxf(mxa[i & 7], x[i]);
        const float mx = fmaxf(fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3])),
                               fmaxf(fmaxf(mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7])));
        const float m_tile = CAP ? mx : mx * sl2;   // running max in log2 units
        const float m_new = fmaxf(m, m_tile);
        float alpha = 1.f;
        bool rescale = false;
        float m_use = m;
        if (m_new > m + 8.f) {
          m_use = m_new;
          rescale = (m != -INFINITY);
          alpha = rescale ? ex2(m - m_new) : 0.f;
        }
        const float mu = (m_use == -INFINITY) ? 0.f : m_use;
        float rsa[8];
#pragma unroll
        for (int a = 0; a < 8; ++a) rsa[a] = 0.f;
        uint32_t pk[BN / 64][32];
#pragma unroll
        for (int i = 0; i < BN; i += 2) {
          // one pair in eight on the FMA pipe: the MUFU unit, 16 exponentials
          // per clock per SM, is what bounds this loop
          float p0, p1;
          if ((i & 15) == 14) {
            const float2 e = ex2_poly2(CAP ? make_float2(x[i] - mu, x[i + 1] - mu)
                                           : make_float2(fmaf(x[i], sl2, -mu), fmaf(x[i + 1], sl2, -mu)));
            p0 = e.x;
            p1 = e.y;
          } else {
            p0 = CAP ? ex2(x[i] - mu) : ex2(fmaf(x[i], sl2, -mu));
            p1 = CAP ? ex2(x[i + 1] - mu) : ex2(fmaf(x[i + 1], sl2, -mu));
          }
          rsa[(i >> 1) & 7] += p0 + p1;
          pk[i >> 6][(i >> 1) & 31] = pack_bf16x2(p0, p1);
        }
        const float rs = ((rsa[0] + rsa[1]) + (rsa[2] + rsa[3])) + ((rsa[4] + rsa[5]) + (rsa[6] + rsa[7]));
        // P (bf16 pairs) over the first BN/2 columns of this S slot
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tmem_st32(scol + c * 32, pk[c]);
        // O must hold P V of every earlier tile of the item before it is
        // rescaled; that is the only case in which the softmax waits for the
        // tensor core.  Seeing S(T) implies P V(T-2) is complete (it was
        // issued before Q K^T(T)), so o_done is at most one phase behind and
        // its parity wait is exact.
        if (__any_sync(0xffffffffu, rescale) && j >= 1) {
          ok = __all_sync(0xffffffffu, mbar_wait(o_done, (T - 1) & 1, tmo, P.status, abort_flag));
          if (!ok) break;
          tc_fence_after();
          const float f = rescale ? alpha : 1.f;
#pragma unroll 1
          for (int c = 0; c < C::DV / 32; ++c) {
            uint32_t o[32];
            tmem_ld32(tmem + lane_off + C::TM_O + c * 32, o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
            tmem_st32(tmem + lane_off + C::TM_O + c * 32, o);
          }
        }
        tmem_wait_st();
        l = (rescale ? l * alpha : l) + rs;
        m = m_use;
        tc_fence_before();
        mbar_arrive(&p_full[T & 1]);
        if (t == 0 && I == 0 && j < 120) mark(128 + j);
      }
      ok = ok && __all_sync(0xffffffffu, mbar_wait(o_final, I & 1, tmo, P.status, abort_flag));
      if (ok) {
        // epilogue: O / l -> bf16, thread t writing row t's DV dims to global
        // memory; then O is free for the next item
        if (t == 0 && I == 0) mark(4);
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* orow = reinterpret_cast<uint4*>(
            P.out + ((static_cast<size_t>(w.b) * S + (in_seq ? qi : 0)) * H + w.h) * D + w.dv_lo);
#pragma unroll 1
        for (int c = 0; c < C::DV / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lane_off + C::TM_O + c * 32, o);
          tmem_wait_ld();
          if (in_seq) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 u;
              u.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
              u.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
              u.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
              u.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
              orow[4 * c + v] = u;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(o_empty);
      T0 += w.ntiles;
      ++I;
    }
  }
  else if (warp == 4) {
    // ------------------------------------------------------------------ producer
    // Each key tile (KCH boxes, ring slots [0, KCH)) and each value tile (VCH
    // boxes, slots [KCH, NSTAGE)) lands under one barrier phase: a phase per
    // box would cap this thread's copy stream far below the L2 rate.  Per
    // item: K(0), then Q (once the previous item's last Q K^T is done with the
    // Q tile), then K(j), V(j-1) in the order the MMA issuer consumes them.
    if (lane == 0) {
      auto load_k = [&](const Item& w, int T, int j) -> bool {
        if (!mbar_wait(ke, (T & 1) ^ 1, tmo, P.status, abort_flag)) return false;
        mbar_arrive_expect_tx(kf, C::KCH * C::SLAB_KV);
        for (int c = 0; c < C::KCH; ++c)
          tma_load_4d(smem + C::OFF_RING + c * C::SLAB_KV, &P.tm_k, kf, c * 64, w.kvh, tile_key(w, j), w.b);
        return true;
      };
      auto load_v = [&](const Item& w, int T, int j) -> bool {
        if (!mbar_wait(ve, (T & 1) ^ 1, tmo, P.status, abort_flag)) return false;
        mbar_arrive_expect_tx(vf, C::VCH * C::SLAB_KV);
        for (int c = 0; c < C::VCH; ++c)
          tma_load_4d(smem + C::OFF_RING + (C::KCH + c) * C::SLAB_KV, &P.tm_v, vf, w.dv_lo + c * 64, w.kvh,
                      tile_key(w, j), w.b);
        return true;
      };
      bool ok = true;
      int T0 = 0, lk = -1, lv = -1, lq = -1;  // last key tile, value tile, Q tile issued
      for (int r = 0, I = 0; r < nrounds && ok; ++r) {
      const int it = item_at(r);
      if (it >= nitems) continue;
        const Item w = item_of(it);
        if (PAD && w.ntiles == 0) continue;  // all padding: nothing to load
        ok = load_k(w, T0, 0);
        if (!ok) break;
        lk = T0;
        ok = mbar_wait(q_empty, (I & 1) ^ 1, tmo, P.status, abort_flag);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
        for (int sl = 0; sl < D / 64; ++sl)
          tma_load_4d(smem + C::OFF_Q + sl * C::SLAB128, &P.tm_q, q_full, sl * 64, w.h, w.q0, w.b);
        lq = I;
        for (int j = 1; j < w.ntiles && ok; ++j) {
          ok = load_k(w, T0 + j, j);
          if (ok) lk = T0 + j;
          if (ok) ok = load_v(w, T0 + j - 1, j - 1);
          if (ok) lv = T0 + j - 1;
        }
        if (ok) ok = load_v(w, T0 + w.ntiles - 1, w.ntiles - 1);
        if (ok) lv = T0 + w.ntiles - 1;
        T0 += w.ntiles;
      ++I;
      }
      // let every issued copy land before the CTA can exit
      if (lq >= 0) mbar_wait(q_full, lq & 1, tmo, P.status, nullptr);
      if (lk >= 0) mbar_wait(kf, lk & 1, tmo, P.status, nullptr);
      if (lv >= 0) mbar_wait(vf, lv & 1, tmo, P.status, nullptr);
    }
  }
  else {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, C::DV, false, true);
      auto qk = [&](int T, bool trace_it, int j) -> bool {
        const uint32_t s_tm = tmem + ((T & 1) ? C::TM_S1 : C::TM_S0);
        if (!mbar_wait(kf, T & 1, tmo, P.status, abort_flag)) return false;
        if (trace_it && j == 0) mark(6);
        tc_fence_after();
        for (int c = 0; c < C::KCH; ++c) {
          const uint32_t kb = sbase + C::OFF_RING + c * C::SLAB_KV;
          const uint32_t qb = sbase + C::OFF_Q + c * C::SLAB128;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bd = smem_desc_sw128(kb + kk * 32, 16, 1024);
            const uint64_t a = smem_desc_sw128(qb + kk * 32, 16, 1024);
            mma_bf16_ss(s_tm, a, bd, idesc_qk, (c | kk) != 0);
          }
        }
        mma_commit(ke);
        mma_commit(&s_full[T & 1]);
        if (trace_it && j < 120) mark(248 + j);
        return true;
      };
      // first: the item's first P V, which overwrites O and so waits until the
      // softmax has read the previous item's O
      auto pv = [&](int T, int I, bool first, bool trace_it, int j) -> bool {
        if (!mbar_wait(&p_full[T & 1], (T >> 1) & 1, tmo, P.status, abort_flag)) return false;
        if (first && !mbar_wait(o_empty, (I & 1) ^ 1, tmo, P.status, abort_flag)) return false;
        const uint32_t p_tm = tmem + ((T & 1) ? C::TM_S1 : C::TM_S0);
        if (!mbar_wait(vf, T & 1, tmo, P.status, abort_flag)) return false;
        tc_fence_after();
        const uint32_t vb = sbase + C::OFF_RING + C::KCH * C::SLAB_KV;
#pragma unroll
        for (int kk = 0; kk < BN / 16; ++kk) {
          // 16 keys x 256 value dims, MN-major: key rows 128 B apart, 8-row groups
          // 1 KB apart, 64-dim boxes one slot apart
          const uint64_t bd = smem_desc_sw128(vb + kk * 16 * 128, C::SLAB_KV, 1024);
          mma_bf16_ts(tmem + C::TM_O, p_tm + kk * 8, bd, idesc_pv, (!first || kk > 0) ? 1u : 0u);
        }
        mma_commit(ve);
        mma_commit(o_done);
        if (trace_it && j < 120) mark(368 + j);
        return true;
      };
      // issue order Q K^T(T), P V(T-1): the S slot of tile T is rewritten by
      // Q K^T(T+2) only after P V(T), which reads P from it, was issued
      bool ok = true;
      int T0 = 0;
      for (int r = 0, I = 0; r < nrounds && ok; ++r) {
      const int it = item_at(r);
      if (it >= nitems) continue;
        const Item w = item_of(it);
        if (PAD && w.ntiles == 0) continue;  // all padding: nothing to multiply
        ok = mbar_wait(q_full, I & 1, tmo, P.status, abort_flag);
        if (!ok) break;
        if (I == 0) mark(3);
        tc_fence_after();
        for (int j = 0; j < w.ntiles && ok; ++j) {
          ok = qk(T0 + j, I == 0, j);
          if (ok && j == w.ntiles - 1) mma_commit(q_empty);  // Q is free once this completes
          if (ok && j >= 1) ok = pv(T0 + j - 1, I, j == 1, I == 0, j - 1);
        }
        if (ok) ok = pv(T0 + w.ntiles - 1, I, w.ntiles == 1, I == 0, w.ntiles - 1);
        mma_commit(o_final);
        T0 += w.ntiles;
      ++I;
      }
      // every MMA issued above has completed before TMEM is released
      mma_commit(drain);
      mbar_wait(drain, 0, tmo, P.status, nullptr);
    }
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0) mark(5);
}

template <int D, int BN, bool CAP, int MODE>
static cudaError_t run_prefill(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s) {
  using C = PrefillShape<D, BN>;
  PrefillKParams P;
  const int kv_rows = MODE == 2 ? pa.KV_S : pa.S;
  if (!encode_tmap_bshd(&P.tm_q, pa.q, pa.B, pa.S, la.H, D, C::BM) ||
      !encode_tmap_bshd(&P.tm_k, pa.kt, pa.B, kv_rows, la.Hkv, D, BN) ||
      !encode_tmap_bshd(&P.tm_v, pa.v, pa.B, kv_rows, la.Hkv, D, BN))
    return cudaErrorInvalidValue;
  P.out = pa.out;
  P.status = pa.status;
  P.timeout_ns = pa.timeout_ns;
  P.B = pa.B;
  P.S = pa.S;
  P.nqt = (pa.S + C::BM - 1) / C::BM;
  P.dv_splits = D / C::DV;
  P.la = la;
  P.trace = pa.trace;
  P.trace_ctas = static_cast<int>(pa.trace_bytes / (kTraceSlots * sizeof(unsigned long long)));
  P.seq_range = pa.seq_range;
  P.q_off = pa.q_off;
  P.KV_S = kv_rows;
  auto kern = prefill_kernel<D, BN, CAP, MODE>;
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  // the shared-memory opt-in is per device: set it once on each device a call runs on
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  // one CTA per SM (the shared memory allows no more), each taking items in turn
  const long long items = static_cast<long long>(P.nqt) * pa.B * la.H * P.dv_splits;
  if (items > (1LL << 31) - 1) return cudaErrorInvalidValue;
  const long long grid = items < sms ? items : sms;
  return launch_pdl(kern, dim3(static_cast<unsigned>(grid)), dim3(192), C::SMEM, s, P);
}

template <int MODE>
static cudaError_t launch_prefill_mode(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s) {
  const bool cap = la.softcap > 0.f;
  if (la.D == 256)
    return cap ? run_prefill<256, 128, true, MODE>(pa, la, s) : run_prefill<256, 128, false, MODE>(pa, la, s);
  if (la.D == 512)
    return cap ? run_prefill<512, 64, true, MODE>(pa, la, s) : run_prefill<512, 64, false, MODE>(pa, la, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_prefill(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s) {
  if (pa.seq_range) return launch_prefill_mode<1>(pa, la, s);
  if (pa.q_off) return launch_prefill_mode<2>(pa, la, s);
  // whole prompts at head_dim 512: two heads of a kv group on an SM pair
  if (prefill_pair_supported(la)) return launch_prefill_pair(pa, la, s);
  return launch_prefill_mode<0>(pa, la, s);
}

}  // namespace gattn
