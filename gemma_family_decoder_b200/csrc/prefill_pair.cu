// Prefill self-attention for head_dim 256 on a pair of SMs (tcgen05 cta_group::2).
//
// A cluster of two CTAs computes the same 128-query tile for two query heads
// of one KV group (GQA/MQA: both heads read the same keys and values).  Every
// tensor-core instruction is a pair MMA with M = 256: each CTA supplies its own
// 128 query rows, and each holds only half of every key/value tile in its
// shared memory (keys [0,64) / [64,128) of a key tile for Q K^T, value dims
// [0,128) / [128,256) for P V), so each SM loads half of the K/V bytes a
// single-SM tile would.  Roles per CTA:
//   warps 0-7  two threads per query row (warp w: TMEM lanes 32*(w%4).., column
//              half w/4): Q-tile prologue (QK-norm + RoPE in place in shared
//              memory), then per KV tile the online softmax on this CTA's S rows
//              (the halves exchange only the row maximum), P written back over
//              its S slot, and the O / l epilogue + TMA store.
//   warp 8     TMA producer for this CTA's Q tile and K/V halves; ring-slot
//              completion is counted on the barriers of CTA 0.
//   warp 9     (CTA 0 only) issues the pair MMAs and their commits, which arrive
//              on the matching barriers of both CTAs.
// The layer definition is the one of the single-SM kernel (prefill.cu).
#include <cuda_bf16.h>

#include "gattn_internal.h"
#include "kernels/common.cuh"
#include "kernels/rowops.cuh"

namespace gattn {

using bf16 = __nv_bfloat16;

namespace {

struct PairShape {
  static constexpr int D = 256;
  static constexpr int BM = 128;                 // query rows per CTA
  static constexpr int BN = 128;                 // keys per KV tile (64 per CTA)
  static constexpr int DV = 256;
  static constexpr int SLAB128 = BM * 128;       // 64 dims x 128 rows (Q tile slab)
  static constexpr int Q_BYTES = (D / 64) * SLAB128;
  static constexpr int SLOT = 16384;             // ring slot
  static constexpr int KBOX = (BN / 2) * 128;    // 64 dims x 64 keys
  static constexpr int VBOX = BN * 128;          // 64 dims x 128 keys
  static constexpr int KSLOTS = 2;               // this CTA's key half: 4 boxes of 8 KB
  static constexpr int VSLOTS = 2;               // this CTA's value half: 2 boxes of 16 KB
  static constexpr int NSTAGE = 8;               // even: 2-slot units never wrap
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_RING = Q_BYTES;
  static constexpr int OFF_BAR = OFF_RING + NSTAGE * SLOT;
  static constexpr int NBAR = 2 * NSTAGE + 12;
  static constexpr int OFF_XCH = OFF_BAR + NBAR * 8;     // row exchange: 2 x 256 floats
  static constexpr int OFF_MISC = OFF_XCH + 512 * 4;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;
  static constexpr uint32_t TM_O = 0;
  static constexpr uint32_t TM_S0 = DV;
  static constexpr uint32_t TM_S1 = DV + BN;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(TM_S1 + BN <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM <= 232448, "shared memory budget");
  static_assert(KSLOTS * SLOT == 4 * KBOX && VSLOTS * SLOT == 2 * VBOX, "slot packing");
};

struct PairParams {
  CUtensorMap tm_q;   // box 64 x 128 rows
  CUtensorMap tm_k;   // box 64 x 64 keys
  CUtensorMap tm_v;   // box 64 x 128 keys
  CUtensorMap tm_o;   // box 64 x 128 rows
  const int* positions;
  uint32_t* status;
  uint64_t timeout_ns;
  int B, S, nqt, pairs_per_group;
  LayerArgs la;
  unsigned long long* trace;  // optional per-CTA timeline (same slots as the single-SM kernel)
  int trace_ctas;
};

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

template <bool CAP>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(320, 1)
    prefill_pair_kernel(const __grid_constant__ PairParams P) {
  using C = PairShape;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                     // CTA 0's copy counts both CTAs' bytes
  uint64_t* empty = bars + C::NSTAGE;        // both CTAs (multicast commits)
  uint64_t* s_full = bars + 2 * C::NSTAGE;   // [2], both CTAs
  uint64_t* p_full = s_full + 2;             // [2], CTA 0: 512 arrivals
  uint64_t* o_done = p_full + 2;             // both CTAs
  uint64_t* q_ready = o_done + 1;            // CTA 0: 512 arrivals
  uint64_t* drain = q_ready + 1;             // CTA 0
  uint64_t* q_full = drain + 1;              // own Q tile
  uint64_t* o_final = q_full + 1;            // both CTAs
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const uint32_t rank = cluster_ctarank();
  const LayerArgs& la = P.la;
  const int H = la.H, S = P.S;
  // work item of the pair: heaviest query tiles first
  int idx = blockIdx.x >> 1;
  const int per_qt = P.B * la.Hkv * P.pairs_per_group;
  const int qt = P.nqt - 1 - idx / per_qt;
  idx %= per_qt;
  const int pg = idx % P.pairs_per_group;
  idx /= P.pairs_per_group;
  const int kvh = idx % la.Hkv;
  const int b = idx / la.Hkv;
  const int h = kvh * la.G + 2 * pg + static_cast<int>(rank);
  const int q0 = qt * C::BM;
  const int kv_hi = min(S, q0 + C::BM);
  const int kv_lo = la.window > 0 ? max(0, q0 - la.window + 1) : 0;
  const int k_first = (kv_lo / C::BN) * C::BN;
  const int ntiles = (kv_hi - k_first + C::BN - 1) / C::BN;
  // KV tiles are visited starting at a tile that differs between the pairs
  // working on one sequence at once, so they do not all read the same L2 lines
  // together (the online softmax is independent of the visiting order)
  const int rot = ntiles > 1 ? (pg * 7 + kvh * 3 + b * 5 + qt) % ntiles : 0;
  auto tile_key = [&](int j) { return k_first + ((j + rot) % ntiles) * C::BN; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int i = 0; i < C::NSTAGE; ++i) {
      mbar_init(&full[i], 2);   // one expect_tx arrival per CTA
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 512);
    }
    mbar_init(o_done, 1);
    mbar_init(q_ready, 512);
    mbar_init(drain, 1);
    mbar_init(q_full, 1);
    mbar_init(o_final, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 8 && lane == 0) {
    tma_prefetch_desc(&P.tm_q);
    tma_prefetch_desc(&P.tm_k);
    tma_prefetch_desc(&P.tm_v);
    tma_prefetch_desc(&P.tm_o);
  }
  if (warp == 9) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers exist before any remote arrival
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint64_t tmo = P.timeout_ns;
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
    trace[2] = ntiles;
  }
  // CTA 0's copies of the barriers that count both CTAs
  auto leader = [&](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0); };

  if (warp < 8) {
    // ------------------------------------------------------------------ softmax
    // two threads per query row: warp w reads TMEM lanes 32*(w%4).. and owns
    // the key / value-dim half hf = w / 4 of every tile
    const int r = (warp & 3) * 32 + lane;     // query row of this thread
    const int hf = warp >> 2;                 // column half
    const int t = threadIdx.x;
    const int qi = q0 + r;
    const bool valid = qi < S;
    const uint32_t lane_off = static_cast<uint32_t>((warp & 3) * 32) << 16;
    // row exchange between the two halves, [2 regions][2 halves][128 rows]: the
    // norm sums use region 1, tile j's maxima region j&1, the final sums region
    // ntiles&1, so no region is rewritten while a slower thread may still read it
    float* xch = reinterpret_cast<float*>(smem + C::OFF_XCH);
    bool ok = __all_sync(0xffffffffu, mbar_wait(q_full, 0, tmo, P.status, abort_flag));
    if (t == 0) mark(6);
    // query prologue in place; RoPE angles computed, not read
    {
      const int h8 = la.rot >> 4, nu = C::D / 8 - 2 * h8;
      float rn = 1.f;
      if (la.qk_norm) {
        const float ss = (ok && valid) ? tile_row_sumsq(smem + C::OFF_Q, C::SLAB128, r, hf * (C::D / 16),
                                                        (hf + 1) * (C::D / 16))
                                       : 0.f;
        xch[256 + hf * 128 + r] = ss;
        named_barrier(1, 256);
        rn = rsqrtf((xch[256 + r] + xch[256 + 128 + r]) / static_cast<float>(C::D) + la.eps);
      }
      if (ok && valid && (la.rot > 0 || la.qk_norm)) {
        int pos = la.rot > 0 ? __ldg(P.positions + static_cast<size_t>(b) * S + qi) : 0;
        if (la.rot > 0 && (pos < 0 || pos >= la.rope_max_pos)) {
          flag_status(P.status, kStatusBounds);
          pos = pos < 0 ? 0 : la.rope_max_pos - 1;
        }
        tile_row_prologue(smem + C::OFF_Q, C::SLAB128, r, pos, la, rn, (hf * h8) >> 1, ((hf + 1) * h8) >> 1,
                          2 * h8 + ((hf * nu) >> 1), 2 * h8 + (((hf + 1) * nu) >> 1));
      }
    }
    fence_proxy_async_smem();
    mbar_arrive_cluster(leader(q_ready));
    if (t == 0) mark(7);

    const float sl2 = la.scale_log2;
    const float kcap = CAP ? la.scale / la.softcap : 0.f;
    const float cap_l2 = CAP ? la.softcap * kLog2e : 0.f;
    const int W = la.window;
    constexpr int HN = C::BN / 2;            // keys per thread per tile
    float m = -INFINITY, l = 0.f;            // l: this thread's half of the row sum
    // every thread reaches the per-tile barrier each iteration; the loop is left
    // by all 256 at once when any wait has failed
    for (int j = 0; j < ntiles; ++j) {
      const bool got = ok && mbar_wait(&s_full[j & 1], (j >> 1) & 1, tmo, P.status, abort_flag);
      if (t == 0 && j < 60) mark(8 + j);
      tc_fence_after();
      const uint32_t scol = tmem + lane_off + ((j & 1) ? C::TM_S1 : C::TM_S0);
      uint32_t rr[HN / 32][32];
#pragma unroll
      for (int c = 0; c < HN / 32; ++c) tmem_ld32(scol + hf * HN + c * 32, rr[c]);
      tmem_wait_ld();

      const int tkey0 = tile_key(j);
      const int key0 = tkey0 + hf * HN;   // first key of this thread's half
      const bool full_tile = (tkey0 + C::BN - 1 <= q0) && (q0 + C::BM <= S) &&
                             (W <= 0 || (q0 + C::BM - 1) - tkey0 < W);
      float x[HN];
#pragma unroll
      for (int i = 0; i < HN; ++i) {
        const float sv = __uint_as_float(rr[i >> 5][i & 31]);
        x[i] = CAP ? cap_l2 * tanh_fast(sv * kcap) : sv;
      }
      if (!full_tile) {
        const int hi = valid ? qi - key0 : -1;
        const int lo = W > 0 ? qi - key0 - W + 1 : -C::BN;
#pragma unroll
        for (int i = 0; i < HN; ++i) x[i] = (i <= hi && i >= lo) ? x[i] : -INFINITY;
      }
      float mxa[8];
#pragma unroll
      for (int a = 0; a < 8; ++a) mxa[a] = x[a];
#pragma unroll
      for (int i = 8; i < HN; ++i) mxa[i & 7] = fmaxf(mxa[i & 7], x[i]);
      float mx = fmaxf(fmaxf(fmaxf(mxa[0], mxa[1]), fmaxf(mxa[2], mxa[3])),
                       fmaxf(fmaxf(mxa[4], mxa[5]), fmaxf(mxa[6], mxa[7])));
      // the row maximum over both halves (the two threads must agree on m)
      float* xm = xch + (j & 1) * 256;
      xm[hf * 128 + r] = mx;
      ok = named_barrier_and(1, 256, got);
      if (!ok) break;
      mx = fmaxf(xm[r], xm[128 + r]);
      const float m_tile = CAP ? mx : mx * sl2;
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
      uint32_t pk[32];
#pragma unroll
      for (int i = 0; i < HN; i += 2) {
        const float p0 = CAP ? ex2(x[i] - mu) : ex2(fmaf(x[i], sl2, -mu));
        const float p1 = CAP ? ex2(x[i + 1] - mu) : ex2(fmaf(x[i + 1], sl2, -mu));
        rsa[(i >> 1) & 7] += p0 + p1;
        pk[i >> 1] = pack_bf16x2(p0, p1);
      }
      const float rs = ((rsa[0] + rsa[1]) + (rsa[2] + rsa[3])) + ((rsa[4] + rsa[5]) + (rsa[6] + rsa[7]));
      // P of this half: bf16 pairs over columns [hf*HN/2, hf*HN/2 + HN/2) of the S slot
      tmem_st32(scol + hf * (HN / 2), pk);
      // seeing S(j) implies P V(j-2) is complete, so o_done's parity wait is exact
      if (__any_sync(0xffffffffu, rescale) && j >= 1) {
        // a failed wait is carried to the next tile's barrier, where all leave together
        ok = __all_sync(0xffffffffu, mbar_wait(o_done, (j - 1) & 1, tmo, P.status, abort_flag));
        tc_fence_after();
        const float f = rescale ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < C::DV / 64; ++c) {   // this thread's half of O's columns
          uint32_t o[32];
          const uint32_t oc = tmem + lane_off + C::TM_O + hf * (C::DV / 2) + c * 32;
          tmem_ld32(oc, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * f);
          tmem_st32(oc, o);
        }
      }
      tmem_wait_st();
      l = (rescale ? l * alpha : l) + rs;
      m = m_use;
      tc_fence_before();
      mbar_arrive_cluster(leader(&p_full[j & 1]));
      if (t == 0 && j < 60) mark(68 + j);
    }
    ok = ok && mbar_wait(o_final, 0, tmo, P.status, abort_flag);
    // the whole row sum: this half's plus the other's
    float* xl = xch + (ntiles & 1) * 256;
    xl[hf * 128 + r] = l;
    ok = named_barrier_and(1, 256, ok);
    const float lt = xl[r] + xl[128 + r];
    if (ok) {
      if (t == 0) mark(4);
      tc_fence_after();
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      uint8_t* orow = smem + C::OFF_Q + r * 128;
#pragma unroll 1
      for (int c = 0; c < C::DV / 64; ++c) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + C::TM_O + hf * (C::DV / 2) + c * 32, o);
        tmem_wait_ld();
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(o[8 * v + 0]) * inv, __uint_as_float(o[8 * v + 1]) * inv);
          u.y = pack_bf16x2(__uint_as_float(o[8 * v + 2]) * inv, __uint_as_float(o[8 * v + 3]) * inv);
          u.z = pack_bf16x2(__uint_as_float(o[8 * v + 4]) * inv, __uint_as_float(o[8 * v + 5]) * inv);
          u.w = pack_bf16x2(__uint_as_float(o[8 * v + 6]) * inv, __uint_as_float(o[8 * v + 7]) * inv);
          const int ch = hf * (C::DV / 16) + 4 * c + v;
          *reinterpret_cast<uint4*>(orow + (ch >> 3) * C::SLAB128 + (((ch & 7) ^ (r & 7)) << 4)) = u;
        }
      }
      fence_proxy_async_smem();
      named_barrier(1, 256);
      if (t == 0) {
#pragma unroll
        for (int sl = 0; sl < C::DV / 64; ++sl)
          tma_store_4d(&P.tm_o, smem + C::OFF_Q + sl * C::SLAB128, sl * 64, h, q0, b);
        bulk_commit();
        bulk_wait_read_all();
      }
    }
  } else if (warp == 8) {
    // ------------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, C::Q_BYTES);
#pragma unroll
      for (int sl = 0; sl < C::D / 64; ++sl)
        tma_load_4d(smem + C::OFF_Q + sl * C::SLAB128, &P.tm_q, q_full, sl * 64, h, q0, b);
      int n = 0;  // 2-slot units issued
      auto wait_slots = [&](int st) -> bool {
        const uint32_t par = ((n / (C::NSTAGE / 2)) & 1) ^ 1;
        return mbar_wait(&empty[st], par, tmo, P.status, abort_flag) &&
               mbar_wait(&empty[st + 1], par, tmo, P.status, abort_flag);
      };
      int nk = 0, nv = 0;
      auto load_k = [&](int key0) -> bool {   // this CTA's 64 keys, all 256 dims
        const int st = (2 * n) % C::NSTAGE;
        if (!wait_slots(st)) return false;
        if (nk < 60) mark(248 + nk);
        ++nk;
        for (int s2 = 0; s2 < 2; ++s2) {
          const uint32_t lb = leader(&full[st + s2]);
          mbar_arrive_expect_tx_cluster(lb, C::SLOT);
          uint8_t* dst = smem + C::OFF_RING + (st + s2) * C::SLOT;
          tma_load_4d_pair(dst, &P.tm_k, lb, (2 * s2) * 64, kvh, key0 + static_cast<int>(rank) * 64, b);
          tma_load_4d_pair(dst + C::KBOX, &P.tm_k, lb, (2 * s2 + 1) * 64, kvh,
                           key0 + static_cast<int>(rank) * 64, b);
        }
        ++n;
        return true;
      };
      auto load_v = [&](int key0) -> bool {   // all 128 keys, this CTA's 128 value dims
        const int st = (2 * n) % C::NSTAGE;
        if (!wait_slots(st)) return false;
        if (nv < 60) mark(308 + nv);
        ++nv;
        for (int s2 = 0; s2 < 2; ++s2) {
          const uint32_t lb = leader(&full[st + s2]);
          mbar_arrive_expect_tx_cluster(lb, C::SLOT);
          tma_load_4d_pair(smem + C::OFF_RING + (st + s2) * C::SLOT, &P.tm_v, lb,
                           static_cast<int>(rank) * 128 + s2 * 64, kvh, key0, b);
        }
        ++n;
        return true;
      };
      bool ok = true;
      for (int j = 0; j < ntiles && ok; ++j) {
        ok = load_k(tile_key(j));
        if (ok && j >= 1) ok = load_v(tile_key(j - 1));
      }
      if (ok) ok = load_v(tile_key(ntiles - 1));
      mbar_wait(q_full, 0, tmo, P.status, nullptr);
      if (!ok) {
        // after a timed-out wait the ring barriers are not trustworthy; give
        // copies issued just before it ~100 us to land before the CTA exits
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 100000) {
        }
      }
    }
  } else if (rank == 0) {
    // ------------------------------------------------------------------ pair MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(256, C::BN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(256, C::DV, false, true);
      constexpr uint16_t both = 0x3;
      int n = 0;
      bool ok = mbar_wait(q_ready, 0, tmo, P.status, abort_flag);
      mark(3);
      tc_fence_after();
      auto wait_full = [&](int st) -> bool {
        const uint32_t par = (n / (C::NSTAGE / 2)) & 1;
        return mbar_wait(&full[st], par, tmo, P.status, abort_flag) &&
               mbar_wait(&full[st + 1], par, tmo, P.status, abort_flag);
      };
      auto qk = [&](int j) -> bool {
        const uint32_t s_tm = tmem + ((j & 1) ? C::TM_S1 : C::TM_S0);
        const int st = (2 * n) % C::NSTAGE;
        if (!wait_full(st)) return false;
        if (j < 60) mark(368 + j);
        tc_fence_after();
        const uint32_t kb = sbase + C::OFF_RING + st * C::SLOT;
#pragma unroll
        for (int c = 0; c < 4; ++c) {           // 64-dim chunk of the key half
          const uint32_t qb = sbase + C::OFF_Q + c * C::SLAB128;
          const uint32_t bb = kb + (c >> 1) * C::SLOT + (c & 1) * C::KBOX;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t a = smem_desc_sw128(qb + kk * 32, 16, 1024);
            const uint64_t bd = smem_desc_sw128(bb + kk * 32, 16, 1024);
            mma_bf16_ss_pair(s_tm, a, bd, idesc_qk, (c | kk) != 0);
          }
        }
        mma_commit_pair(&empty[st], both);
        mma_commit_pair(&empty[st + 1], both);
        mma_commit_pair(&s_full[j & 1], both);
        ++n;
        if (j < 60) mark(128 + j);
        return true;
      };
      auto pv = [&](int i) -> bool {
        if (!mbar_wait(&p_full[i & 1], (i >> 1) & 1, tmo, P.status, abort_flag)) return false;
        const uint32_t p_tm = tmem + ((i & 1) ? C::TM_S1 : C::TM_S0);
        const int st = (2 * n) % C::NSTAGE;
        if (!wait_full(st)) return false;
        if (i < 60) mark(428 + i);
        tc_fence_after();
        const uint32_t vb = sbase + C::OFF_RING + st * C::SLOT;
#pragma unroll
        for (int kk = 0; kk < C::BN / 16; ++kk) {
          // 16 keys x 128 value dims per CTA, MN-major: 64-dim boxes one slot apart
          const uint64_t bd = smem_desc_sw128(vb + kk * 16 * 128, C::SLOT, 1024);
          mma_bf16_ts_pair(tmem + C::TM_O, p_tm + kk * 8, bd, idesc_pv, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_pair(&empty[st], both);
        mma_commit_pair(&empty[st + 1], both);
        mma_commit_pair(o_done, both);
        ++n;
        if (i < 60) mark(188 + i);
        return true;
      };
      for (int j = 0; j < ntiles && ok; ++j) {
        ok = qk(j);
        if (ok && j >= 1) ok = pv(j - 1);
      }
      if (ok) pv(ntiles - 1);
      mma_commit_pair(o_final, both);
      mma_commit_pair(drain, 0x1);
      mbar_wait(drain, 0, tmo, P.status, nullptr);
    }
  }
  __syncwarp();
  tc_fence_before();
  // neither CTA leaves (or frees TMEM) while the pair's MMAs may still touch it
  cluster_sync();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
  if (threadIdx.x == 0) mark(5);
}

bool prefill_pair_supported(const LayerArgs& la) { return la.D == 256 && la.G % 2 == 0; }

cudaError_t launch_prefill_pair(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s) {
  using C = PairShape;
  PairParams P;
  if (!encode_tmap_bshd(&P.tm_q, pa.q, pa.B, pa.S, la.H, C::D, C::BM) ||
      !encode_tmap_bshd(&P.tm_k, pa.kt, pa.B, pa.S, la.Hkv, C::D, C::BN / 2) ||
      !encode_tmap_bshd(&P.tm_v, pa.v, pa.B, pa.S, la.Hkv, C::D, C::BN) ||
      !encode_tmap_bshd(&P.tm_o, pa.out, pa.B, pa.S, la.H, C::D, C::BM))
    return cudaErrorInvalidValue;
  P.positions = pa.positions;
  P.status = pa.status;
  P.timeout_ns = pa.timeout_ns;
  P.B = pa.B;
  P.S = pa.S;
  P.nqt = (pa.S + C::BM - 1) / C::BM;
  P.pairs_per_group = la.G / 2;
  P.la = la;
  P.trace = pa.trace;
  P.trace_ctas = static_cast<int>(pa.trace_bytes / (512 * sizeof(unsigned long long)));
  const bool cap = la.softcap > 0.f;
  auto kern = cap ? prefill_pair_kernel<true> : prefill_pair_kernel<false>;
  static bool attr_set[2] = {false, false};
  if (!attr_set[cap]) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[cap] = true;
  }
  const long long grid = 2LL * P.nqt * pa.B * la.Hkv * P.pairs_per_group;
  kern<<<static_cast<unsigned>(grid), 320, C::SMEM, s>>>(P);
  return cudaGetLastError();
}

}  // namespace gattn
