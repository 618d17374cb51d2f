// Prefill self-attention for head_dim 512 on pairs of SMs (tcgen05 cta_group::2).
//
// At head_dim 512 a Q K^T instruction with A = Q (4 KB per K-step) read from
// shared memory needs more operand bandwidth than one SM's shared memory
// delivers at N = 64, and a 128-query tile's fp32 O over all 512 value dims
// would fill tensor memory; so the single-SM kernel runs 64-key tiles and
// splits the value dims over two work items, at well under the tensor rate.
// Here a cluster of two CTAs works on two query heads of one kv group (both
// read the same keys and values) for one 128-query tile and one 256-wide half
// of the value dims.  Every tensor instruction is a pair MMA with M = 256:
// each CTA supplies its own 128 query rows, and each holds only its half of
// every key tile (64 of its 128 keys, for Q K^T) and of every value tile (128
// of the 256 value dims, for P V); the hardware shares the B operands between
// the two SMs.  Per 128-key tile each SM reads 320 KB of shared memory
// (operands and landing copies) against 3072 cycles of MMA: the tensor core,
// not shared memory, sets the pace.
//
// Roles per CTA:
//   warps 0-3  thread t = query row t of this CTA's head: per tile, S from
//              tensor memory -> scale (and softcap) -> mask on boundary tiles
//              -> online softmax with lazy rescale -> P (bf16) over its S slot;
//              at the end of an item O / l -> bf16 to global memory.
//   warp 4     TMA producer: this CTA's Q tile (128 x 512) and its halves of
//              the key / value tiles into a ring of three 32 KB units (one
//              barrier phase each: a single thread's copy stream is limited by
//              phases, not bytes), each unit's bytes counted on the first
//              CTA's barrier.
//   warp 5     (first CTA only) issues the pair MMAs and their commits, which
//              arrive on the matching barriers of both CTAs.
//   warp 6     a second TMA producer (alternate ring units).
// Clusters are persistent and take items heaviest first in zig-zag rounds.
//
// Layer definition: KerasFormers "Gemma 4" (What changed: global layers with
// head dim 512, K=V, plain-weight RMSNorm, zero-padded partial rotation); the
// queries and keys arrive normed and rotated from the prologue kernel.
#include <cuda_bf16.h>

#include "gattn_internal.h"
#include "kernels/common.cuh"

namespace gattn {

using bf16 = __nv_bfloat16;

namespace {

template <int D_>
struct PairShape {
  static constexpr int D = D_;
  static constexpr int BM = 128;                   // query rows per CTA
  static constexpr int BN = 128;                   // keys per tile (64 per CTA for Q K^T)
  static constexpr int DV = 256;                   // value dims per item (128 per CTA for P V)
  static_assert(D == 256 || D == 512, "head_dim 256 or 512");
  static constexpr int QBOX = BM * 128;            // 64 dims x 128 rows, 128-byte swizzle
  static constexpr int Q_BYTES = (D / 64) * QBOX;  // 128 KB
  static constexpr int KBOX = 8192;                // key box: 64 dims x this CTA's 64 keys
  static constexpr int VBOX = 16384;               // value box: 64 dims x 128 keys
  static constexpr int UNIT = 4 * KBOX;            // one barrier phase: 32 KB per CTA
  static constexpr int DVS = D / 256;              // work items per query tile and head pair (value halves)
  static constexpr int NUNIT = (232448 - Q_BYTES - 1536) / UNIT;  // ring: 3 units at D 512, 5 at D 256
  static constexpr int KUNITS = D / 256;           // units of a key tile (256 dims each)
  static constexpr int VUNITS = 1;                 // units of a value tile (this CTA's 128 dims)
  static_assert(2 * VBOX == UNIT, "a value tile fills one unit");
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NUNIT * UNIT;
  static constexpr int NBAR = 2 * NUNIT + 16;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;  // + slack to align the base to 1 KB
  static constexpr uint32_t TM_O = 0;
  static constexpr uint32_t TM_S0 = DV;
  static constexpr uint32_t TM_S1 = DV + BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(TM_S1 + BN <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
};

struct PairParams {
  CUtensorMap tm_q;  // q~ [B][S][H][512], box 64 x 128 rows
  CUtensorMap tm_k;  // k~ [B][S][Hkv][512], box 64 x 64 keys
  CUtensorMap tm_v;  // v (raw k when K=V), box 64 x 128 keys
  bf16* out;
  uint32_t* status;
  uint64_t timeout_ns;
  int B, S, nqt, npairs;  // npairs = G / 2 head pairs per kv head
  LayerArgs la;
  unsigned long long* trace;  // optional per-CTA timeline (512 slots each), or null
  int trace_ctas;
};

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

template <int D, bool CAP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(224, 1)
    prefill_pair_kernel(const __grid_constant__ PairParams P) {
  using C = PairShape<D>;
  constexpr int BN = C::BN;
  extern __shared__ uint8_t smem_raw[];
  // identical kernels, so the aligned offsets agree between the two CTAs
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                    // [NUNIT] first CTA: both CTAs' bytes of a unit
  uint64_t* empty = bars + C::NUNIT;        // [NUNIT] both CTAs: the unit's MMAs are done
  uint64_t* s_full = bars + 2 * C::NUNIT;   // [2] both: S ready in its TMEM slot
  uint64_t* p_full = s_full + 2;            // [2] first CTA: P written (one arrival per softmax warp)
  uint64_t* o_done = p_full + 2;            // both: one phase per P V
  uint64_t* q_full = o_done + 1;            // first CTA: both Q tiles landed
  uint64_t* q_empty = q_full + 1;           // both: the item's last Q K^T is done
  uint64_t* o_final = q_empty + 1;          // both: the item's last P V is done
  uint64_t* o_empty = o_final + 1;          // first CTA: both softmaxes read O (one arrival per warp)
  uint64_t* drain = o_empty + 1;            // first CTA
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t rank = cluster_ctarank();
  const LayerArgs& la = P.la;
  const int H = la.H, S = P.S;
  const int per_qt = P.B * la.Hkv * P.npairs * C::DVS;
  const int nitems = P.nqt * per_qt;
  struct Item {
    int qt, dvs, h, b, kvh, q0, dv_lo, k_first, ntiles, rot;
  };
  auto item_of = [&](int it) {
    Item w;
    w.qt = P.nqt - 1 - it / per_qt;
    int idx = it % per_qt;
    w.dvs = idx % C::DVS;
    idx /= C::DVS;
    const int pg = idx % P.npairs;
    idx /= P.npairs;
    w.kvh = idx % la.Hkv;
    w.b = idx / la.Hkv;
    w.h = w.kvh * la.G + 2 * pg + static_cast<int>(rank);
    w.q0 = w.qt * C::BM;
    w.dv_lo = w.dvs * C::DV;
    const int kv_hi = min(S, w.q0 + C::BM);
    const int kv_lo = la.window > 0 ? max(0, w.q0 - la.window + 1) : 0;
    w.k_first = (kv_lo / BN) * BN;
    w.ntiles = (kv_hi - w.k_first + BN - 1) / BN;
    // items reading one sequence at once start at different key tiles, so
    // they do not all read the same L2 lines together (the order is free; it
    // follows the pair's first head, so a layout of the same heads over more
    // kv heads visits the same tiles in the same order)
    w.rot = w.ntiles > 1 ? ((w.h - static_cast<int>(rank)) * 7 + w.b * 5 + w.qt + w.dvs * 11) % w.ntiles : 0;
    return w;
  };
  auto tile_key = [&](const Item& w, int j) { return w.k_first + ((j + w.rot) % w.ntiles) * BN; };
  const int NC = static_cast<int>(gridDim.x >> 1), cid = static_cast<int>(blockIdx.x >> 1);
  const int nrounds = (nitems + NC - 1) / NC;
  auto item_at = [&](int r) { return r * NC + ((r & 1) ? NC - 1 - cid : cid); };
  auto leader = [&](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NUNIT; ++i) {
      mbar_init(&full[i], 2);  // one expect_tx arrival per CTA
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 8);
    }
    mbar_init(o_done, 1);
    mbar_init(q_full, 2);
    mbar_init(q_empty, 1);
    mbar_init(o_final, 1);
    mbar_init(o_empty, 8);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if ((warp == 4 || warp == 6) && lane == 0) {
    tma_prefetch_desc(&P.tm_q);
    tma_prefetch_desc(&P.tm_k);
    tma_prefetch_desc(&P.tm_v);
  }
  if (warp == 5) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();  // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  pdl_wait();          // the prologue's q~ and k~ are complete
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = P.timeout_ns;
  // optional timeline of each traced CTA's first item (debug aid, off unless a
  // trace buffer is set): [0] start (ns), [1] SM id, [2] rank, [3] items, [4]
  // tiles of the first item; per tile j < 120: [8+j] S seen by the softmax,
  // [128+j] P written, [248+j] Q K^T issued, [368+j] P V issued
  unsigned long long* trace = (P.trace && static_cast<int>(blockIdx.x) < P.trace_ctas)
                                  ? P.trace + static_cast<size_t>(blockIdx.x) * 512 : nullptr;
  const uint64_t t_start = globaltimer_ns();
  auto mark = [&](int slot) {
    if (trace) trace[slot] = globaltimer_ns() - t_start;
  };
  if (trace && threadIdx.x == 0) {
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    trace[0] = t_start;
    trace[1] = smid;
    trace[2] = rank;
    int n = 0;
    for (int r = 0; r < nrounds; ++r) n += item_at(r) < nitems;
    trace[3] = n;
    trace[4] = item_of(item_at(0)).ntiles;
  }

  if (warp < 4) {
    // ------------------------------------------------------------------ softmax
    const int t = threadIdx.x;
    const uint32_t lane_off = static_cast<uint32_t>(warp * 32) << 16;
    const float sl2 = la.scale_log2;
    const float kcap = CAP ? la.scale / la.softcap : 0.f;
    const float cap_l2 = CAP ? la.softcap * kLog2e : 0.f;
    const int W = la.window;
    const uint32_t p_full_l[2] = {leader(&p_full[0]), leader(&p_full[1])};
    const uint32_t o_empty_l = leader(o_empty);
    bool ok = true;
    int T0 = 0;
    for (int r = 0, I = 0; r < nrounds && ok; ++r) {
      const int it = item_at(r);
      if (it >= nitems) continue;
      const Item w = item_of(it);
      const int qi = w.q0 + t;
      const bool in_seq = qi < S;
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
        const bool full_tile = (key0 + BN - 1 <= w.q0) && (w.q0 + C::BM <= S) &&
                               (W <= 0 || (w.q0 + C::BM - 1) - key0 < W);
        float x[BN];
#pragma unroll
        for (int i = 0; i < BN; ++i) {
          const float sv = __uint_as_float(rr[i >> 5][i & 31]);
          x[i] = CAP ? cap_l2 * tanh_fast(sv * kcap) : sv;
        }
        if (!full_tile) {
          const int hi = in_seq ? qi - key0 : -1;             // visible iff i <= hi
          const int lo = W > 0 ? qi - key0 - W + 1 : -BN;      // and i >= lo
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
        const float m_tile = CAP ? mx : mx * sl2;  // running max in log2 units
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
          // one pair in eight on the FMA pipe (the MUFU unit bounds this loop)
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
#pragma unroll
        for (int c = 0; c < BN / 64; ++c) tmem_st32(scol + c * 32, pk[c]);
        // O must hold P V of every earlier tile before it is rescaled (seeing
        // S(T) implies P V(T-2) completed: o_done is at most one phase behind)
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
        // the warp's tensor-memory stores are complete (wait::st is warp-wide):
        // one cluster-scope arrival per warp instead of one fence per thread
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(p_full_l[T & 1]);
        if (t == 0 && I == 0 && j < 120) mark(128 + j);
      }
      ok = ok && __all_sync(0xffffffffu, mbar_wait(o_final, I & 1, tmo, P.status, abort_flag));
      if (ok) {
        // epilogue: O / l -> bf16, thread t writing row t's 256 dims
        tc_fence_after();
        const float inv = l > 0.f ? 1.f / l : 0.f;
        uint4* orow = reinterpret_cast<uint4*>(
            P.out + ((static_cast<size_t>(w.b) * S + (in_seq ? qi : 0)) * H + w.h) * C::D + w.dv_lo);
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
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(o_empty_l);
      T0 += w.ntiles;
      ++I;
    }
  } else if (warp == 4 || warp == 6) {
    // ------------------------------------------------------------------ producers
    // Units are issued in the order the MMAs consume them: the key units of
    // tile 0, this CTA's Q tile, then per tile j the key units of j and the
    // value unit of j - 1.  A key unit holds this CTA's 64 keys of the tile at
    // 256 dims (four boxes); a value unit all 128 keys at this CTA's 128 value
    // dims (two boxes).  Two threads in two warps issue alternate units (and
    // the first the Q tiles): one thread's copy stream is limited by a fixed
    // cost per barrier phase, which a second issuing thread halves.
    if (lane == 0) {
      const int pid = warp == 4 ? 0 : 1;
      int n = 0;  // units of the sequence so far (either thread's)
      auto acquire = [&](int& u) -> bool {
        u = n % C::NUNIT;
        return mbar_wait(&empty[u], ((n / C::NUNIT) & 1) ^ 1, tmo, P.status, abort_flag);
      };
      auto load_k = [&](const Item& w, int j) -> bool {
        const int key = tile_key(w, j) + static_cast<int>(rank) * (BN / 2);
        for (int ku = 0; ku < C::KUNITS; ++ku, ++n) {
          if ((n & 1) != pid) continue;
          int u;
          if (!acquire(u)) return false;
          const uint32_t lb = leader(&full[u]);
          mbar_arrive_expect_tx_cluster(lb, C::UNIT);
          uint8_t* dst = smem + C::OFF_RING + u * C::UNIT;
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tma_load_4d_pair(dst + c * C::KBOX, &P.tm_k, lb, ku * 256 + c * 64, w.kvh, key, w.b);
        }
        return true;
      };
      auto load_v = [&](const Item& w, int j) -> bool {
        const int dv = w.dv_lo + static_cast<int>(rank) * (C::DV / 2);
        for (int vu = 0; vu < C::VUNITS; ++vu, ++n) {
          if ((n & 1) != pid) continue;
          int u;
          if (!acquire(u)) return false;
          const uint32_t lb = leader(&full[u]);
          mbar_arrive_expect_tx_cluster(lb, C::UNIT);
          uint8_t* dst = smem + C::OFF_RING + u * C::UNIT;
          const int key = tile_key(w, j);
          tma_load_4d_pair(dst, &P.tm_v, lb, dv, w.kvh, key, w.b);
          tma_load_4d_pair(dst + C::VBOX, &P.tm_v, lb, dv + 64, w.kvh, key, w.b);
        }
        return true;
      };
      const uint32_t q_full_l = leader(q_full);
      bool ok = true;
      int lq = -1;  // last Q tile issued
      for (int r = 0, I = 0; r < nrounds && ok; ++r) {
        const int it = item_at(r);
        if (it >= nitems) continue;
        const Item w = item_of(it);
        ok = load_k(w, 0);
        if (!ok) break;
        if (pid == 0) {
          ok = mbar_wait(q_empty, (I & 1) ^ 1, tmo, P.status, abort_flag);
          if (!ok) break;
          mbar_arrive_expect_tx_cluster(q_full_l, C::Q_BYTES);
#pragma unroll 1
          for (int c = 0; c < C::D / 64; ++c)
            tma_load_4d_pair(smem + C::OFF_Q + c * C::QBOX, &P.tm_q, q_full_l, c * 64, w.h, w.q0, w.b);
          lq = I;
        }
        for (int j = 1; j < w.ntiles && ok; ++j) {
          ok = load_k(w, j);
          if (ok) ok = load_v(w, j - 1);
        }
        if (ok) ok = load_v(w, w.ntiles - 1);
        ++I;
      }
      // every copy issued lands before the CTA can exit: the MMAs that read
      // the last NUNIT units (and the last Q tile) completed, so did their copies
      for (int k = n - C::NUNIT > 0 ? n - C::NUNIT : 0; k < n; ++k)
        if ((k & 1) == pid) mbar_wait(&empty[k % C::NUNIT], (k / C::NUNIT) & 1, tmo, P.status, nullptr);
      if (lq >= 0) mbar_wait(q_empty, lq & 1, tmo, P.status, nullptr);
    }
  } else if (rank == 0) {
    // ------------------------------------------------------------------ pair MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(256, BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(256, C::DV, false, true);
      constexpr uint16_t both = 0x3;
      int n = 0;  // units consumed
      auto take = [&](int& u) -> bool {
        u = n % C::NUNIT;
        if (!mbar_wait(&full[u], (n / C::NUNIT) & 1, tmo, P.status, abort_flag)) return false;
        tc_fence_after();
        return true;
      };
      auto qk = [&](int T, bool tr) -> bool {
        const uint32_t s_tm = tmem + ((T & 1) ? C::TM_S1 : C::TM_S0);
        for (int ku = 0; ku < C::KUNITS; ++ku) {
          int u;
          if (!take(u)) return false;
          const uint32_t kb = sbase + C::OFF_RING + u * C::UNIT;
#pragma unroll
          for (int s2 = 0; s2 < 4; ++s2) {
            const int dc = 4 * ku + s2;  // 64-dim chunk
            const uint32_t qb = sbase + C::OFF_Q + dc * C::QBOX;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_bf16_ss_pair(s_tm, smem_desc_sw128(qb + kk * 32, 16, 1024),
                               smem_desc_sw128(kb + s2 * C::KBOX + kk * 32, 16, 1024), idesc_qk, (dc | kk) != 0);
          }
          mma_commit_pair(&empty[u], both);
          ++n;
        }
        mma_commit_pair(&s_full[T & 1], both);
        if (tr && T < 120) mark(248 + T);
        return true;
      };
      // first: the item's first P V, which overwrites O and so waits until
      // both softmaxes have read the previous item's O
      auto pv = [&](int T, int I, bool first, bool tr) -> bool {
        if (!mbar_wait(&p_full[T & 1], (T >> 1) & 1, tmo, P.status, abort_flag)) return false;
        if (first && !mbar_wait(o_empty, (I & 1) ^ 1, tmo, P.status, abort_flag)) return false;
        const uint32_t p_tm = tmem + ((T & 1) ? C::TM_S1 : C::TM_S0);
        for (int vu = 0; vu < C::VUNITS; ++vu) {
          int u;
          if (!take(u)) return false;
          const uint32_t vb = sbase + C::OFF_RING + u * C::UNIT;
#pragma unroll
          for (int kk = 0; kk < BN / 16; ++kk) {
            // 16 keys x this CTA's 128 value dims, MN-major: key rows 128 B
            // apart, 8-row groups 1 KB apart, the two 64-dim boxes one box apart
            const uint64_t bd = smem_desc_sw128(vb + kk * 16 * 128, C::VBOX, 1024);
            mma_bf16_ts_pair(tmem + C::TM_O, p_tm + kk * 8, bd, idesc_pv, (!first || kk > 0) ? 1u : 0u);
          }
          mma_commit_pair(&empty[u], both);
          ++n;
        }
        mma_commit_pair(o_done, both);
        if (tr && T < 120) mark(368 + T);
        return true;
      };
      bool ok = true;
      int T0 = 0;
      for (int r = 0, I = 0; r < nrounds && ok; ++r) {
        const int it = item_at(r);
        if (it >= nitems) continue;
        const Item w = item_of(it);
        // the item's Q K^T needs both CTAs' Q tiles; its first key units may land earlier
        ok = mbar_wait(q_full, I & 1, tmo, P.status, abort_flag);
        if (!ok) break;
        tc_fence_after();
        for (int j = 0; j < w.ntiles && ok; ++j) {
          ok = qk(T0 + j, I == 0);
          if (ok && j == w.ntiles - 1) mma_commit_pair(q_empty, both);  // Q is free once this completes
          if (ok && j >= 1) ok = pv(T0 + j - 1, I, j == 1, I == 0);
        }
        if (ok) ok = pv(T0 + w.ntiles - 1, I, w.ntiles == 1, I == 0);
        mma_commit_pair(o_final, both);
        T0 += w.ntiles;
        ++I;
      }
      // every MMA issued above has completed before tensor memory is released
      mma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, tmo, P.status, nullptr);
    }
  }
  __syncwarp();
  tc_fence_before();
  // neither CTA leaves (or frees tensor memory) while the pair's MMAs or the
  // other CTA's arrivals may still reach it
  cluster_sync_all();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

// head_dim 512 only: at head_dim 256 the single-SM kernel holds both tiles'
// operands within shared memory's bandwidth, and the pair measured slower
// (Gemma-1 MQA prefill 738 against 920 TFLOP/s, Gemma-3 global 1087 against 1310)
bool prefill_pair_supported(const LayerArgs& la) { return la.D == 512 && la.G % 2 == 0; }

template <int D>
static cudaError_t run_pair(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s) {
  using C = PairShape<D>;
  PairParams P;
  if (!encode_tmap_bshd(&P.tm_q, pa.q, pa.B, pa.S, la.H, C::D, C::BM) ||
      !encode_tmap_bshd(&P.tm_k, pa.kt, pa.B, pa.S, la.Hkv, C::D, C::BN / 2) ||
      !encode_tmap_bshd(&P.tm_v, pa.v, pa.B, pa.S, la.Hkv, C::D, C::BN))
    return cudaErrorInvalidValue;
  P.out = pa.out;
  P.status = pa.status;
  P.timeout_ns = pa.timeout_ns;
  P.B = pa.B;
  P.S = pa.S;
  P.nqt = (pa.S + C::BM - 1) / C::BM;
  P.npairs = la.G / 2;
  P.la = la;
  P.trace = pa.trace;
  P.trace_ctas = static_cast<int>(pa.trace_bytes / (512 * sizeof(unsigned long long)));
  const bool cap = la.softcap > 0.f;
  auto kern = cap ? prefill_pair_kernel<D, true> : prefill_pair_kernel<D, false>;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  // per device: the shared-memory opt-in and how many pairs can be resident
  constexpr int kMaxDev = 64;
  static int max_clusters[kMaxDev][2] = {};  // per instance (D fixed here), per softcap
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  int& mc = max_clusters[dev][cap ? 1 : 0];
  if (mc == 0) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t qc = {};
    qc.gridDim = dim3(2);
    qc.blockDim = dim3(224);
    qc.dynamicSmemBytes = C::SMEM;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &qc);
    if (e != cudaSuccess) return e;
    if (n < 1) return cudaErrorInvalidConfiguration;
    mc = n;
  }
  const long long items = static_cast<long long>(P.nqt) * pa.B * la.Hkv * P.npairs * C::DVS;
  if (items > (1LL << 31) - 1) return cudaErrorInvalidValue;
  const long long nc = items < mc ? items : mc;
  return launch_pdl(kern, dim3(static_cast<unsigned>(2 * nc)), dim3(224), C::SMEM, s, P);
}

cudaError_t launch_prefill_pair(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s) {
  if (!prefill_pair_supported(la) || pa.seq_range || pa.q_off) return cudaErrorInvalidValue;
  return run_pair<512>(pa, la, s);
}

}  // namespace gattn
