// Split-KV decode on CUDA cores for small query groups: 1, 2 or 4 query heads
// per key/value head (the Gemma 4 local layer: 16 query heads on 8 kv heads,
// separate K and V caches, full RoPE), for every layer the tensor-core decode
// does not take.  Per query head and key the work is a few multiply-adds per
// byte of cache, so the kernel is built to keep HBM busy:
//
// * Persistent: one CTA per SM.  The (sequence, chunk) work items, sequence-
//   major, are cut into equal contiguous ranges, one per CTA; the chunks of one
//   sequence inside a range form a segment, streamed as one key range.
// * A tile is 32 KB of consecutive cache rows (all kv heads of TP positions),
//   moved by one bulk copy (and the value rows by a second, and the rows of
//   the RoPE table for its positions by a third) into a ring of stages; the
//   last warp to finish with a stage refills it.
// * Warp w (of 8) serves kv head w % Hkv and, of every tile, the positions
//   sub + SUB r (sub = w / Hkv, SUB = 8 / Hkv).  Lane l owns dims 4l + 128c + e
//   (c < D/128, e < 4), so the two dims of a rotate-half pair sit in one lane
//   whenever half the rotated slice is 128 dims or more; for smaller slices
//   the partner comes from lane l ^ (R/8).
// * The logits of a warp's rows of a tile (rows x heads, at most 32) are summed
//   over the lanes by one transposing butterfly (31 shuffles for 32 sums), the
//   online softmax runs on those, and P V reads the probabilities back from a
//   per-warp scratch.
//
// * An int8 cache (Q8) keeps the tile's rows and positions but half the bytes,
//   with more stages in flight.  Each warp copies the fp32 scales of its own
//   rows of a tile (4-byte asynchronous copies, one commit group per tile,
//   NST tiles ahead); the key scale multiplies the reduced logit (and, squared,
//   the QK-norm sum of squares), the value scale the probability that P V reads.
//
// Output: the same (m, l, O) partial per (b, head, split) as the other decode
// kernels, split = chunk * SUB + sub, merged by decode_combine_kernel.  Every
// split slot of every sequence is written once: a real partial by the segment
// that starts there, an empty one (m = -inf, l = 0) otherwise.
#include <cuda_bf16.h>

#include <type_traits>

#include "gattn_internal.h"
#include "kernels/common.cuh"
#include "kernels/rowops.cuh"

namespace gattn {

namespace {

constexpr int kSW = 8;                  // compute warps
constexpr int kTileBytes = 32768;       // bf16 cache bytes per tile (keys; values as many); int8: half
constexpr int kTabBytes = 8192;         // RoPE table rows of a tile, staged when they fit

constexpr unsigned kFull = 0xffffffffu;

constexpr int ilog2(int n) { return n <= 1 ? 0 : 1 + ilog2(n >> 1); }

template <int D, int G, bool KEQV, bool Q8>
struct SimtShape {
  static constexpr int NC = D / 128;                 // 4-dim groups per lane
  static constexpr int ES = Q8 ? 1 : 2;              // bytes per cached value
  static constexpr int ROWS = kTileBytes / (2 * D);  // cache rows per tile
  static constexpr int KT = ROWS * D * ES;           // bytes of a tile's key rows (value rows as many)
  static constexpr int RPW = ROWS / kSW;             // rows per warp per tile
  static constexpr int NV = RPW * G;                 // logits per warp per tile
  static constexpr int LOGNV = ilog2(NV);
  static constexpr int LOGG = ilog2(G);
  static constexpr int OFF_TAB = KEQV ? KT : 2 * KT;  // the tile's RoPE table rows
  static constexpr int STAGE = OFF_TAB + kTabBytes;
  static constexpr int NST = Q8 ? (KEQV ? 8 : 5) : (KEQV ? 5 : 3);
  static constexpr int OFF_BAR = NST * STAGE;
  static constexpr int OFF_MISC = OFF_BAR + 2 * NST * 8;
  static constexpr int OFF_SCR = OFF_MISC + 16;      // per warp: p [32], 1/rms [8]
  static constexpr int SCR_FLOATS = 40;
  static constexpr int OFF_SSC = OFF_SCR + kSW * SCR_FLOATS * 4;  // Q8, per warp: [NST][K, V][RPW] scales
  static constexpr int SSC_FLOATS = Q8 ? NST * 2 * RPW : 0;
  static constexpr int SMEM = OFF_SSC + kSW * SSC_FLOATS * 4 + 128;  // + slack to align the base
  static_assert(NV >= 2 && NV <= 32 && (NV & (NV - 1)) == 0, "logits per warp tile");
  static_assert(G * NC * 4 <= 32, "accumulator registers per lane");
  static_assert(RPW <= 8, "norm scratch");
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

struct SimtParams {
  DecodeArgs da;
  LayerArgs la;
  int nch;  // chunks per sequence (da.nsplit = nch * SUB)
  uint64_t timeout_ns;
};

// One segment of a CTA's range: sequence b, chunks [c0, c1], cache positions
// [ps, pe) (empty when ps >= pe).
struct Seg {
  int b, c0, c1, ps, pe, L;
  bool bad_len;
};

__device__ __forceinline__ Seg segment(const SimtParams& P, int b, long long i0, long long i1) {
  const DecodeArgs& da = P.da;
  Seg s;
  s.b = b;
  s.c0 = (b == static_cast<int>(i0 / P.nch)) ? static_cast<int>(i0 % P.nch) : 0;
  s.c1 = (b == static_cast<int>((i1 - 1) / P.nch)) ? static_cast<int>((i1 - 1) % P.nch) : P.nch - 1;
  s.L = __ldg(da.seq_lens + b);
  s.bad_len = s.L < 1 || s.L > da.max_len;
  if (s.bad_len) {
    s.ps = s.pe = 0;
  } else {
    const int lo = P.la.window > 0 ? max(0, s.L - P.la.window) : 0;
    s.ps = lo + s.c0 * da.chunk;
    s.pe = min(s.L, lo + (s.c1 + 1) * da.chunk);
  }
  return s;
}

// Walks the tiles of a CTA's range in order: segment after segment, TP
// positions at a time.  `next` yields the sequence, the first cache position
// and the positions of the following tile, or false past the last one.
struct TileCursor {
  int b, b_last, p0, pe, TP;
  long long i0, i1;
  __device__ __forceinline__ void init(const SimtParams& P, long long i0_, long long i1_, int tp) {
    i0 = i0_;
    i1 = i1_;
    TP = tp;
    b = static_cast<int>(i0 / P.nch) - 1;
    b_last = static_cast<int>((i1 - 1) / P.nch);
    p0 = pe = 0;
  }
  __device__ __forceinline__ bool next(const SimtParams& P, int* tb, int* tp0, int* tn) {
    while (p0 >= pe) {
      if (b >= b_last) return false;
      ++b;
      const Seg sg = segment(P, b, i0, i1);
      p0 = sg.ps;
      pe = sg.pe;
    }
    *tb = b;
    *tp0 = p0;
    *tn = min(TP, pe - p0);
    p0 += TP;
    return true;
  }
};

// Sum of v[i] over the 32 lanes for every i < NV.  Step s exchanges across
// lane bit s: a lane with that bit set keeps the upper half of its entries.
// The lane ends with the total of entry idx = sum_s bit_s(lane) * NV >> (s+1),
// held in the 32 / NV lanes that share those bits.
template <int NV>
__device__ __forceinline__ float transpose_sum(float (&v)[NV], int lane) {
  constexpr int LOG = ilog2(NV);
#pragma unroll
  for (int s = 0; s < LOG; ++s) {
    const int w = NV >> (s + 1);
    const bool up = (lane >> s) & 1;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float send = up ? v[i] : v[i + w];
      const float keep = up ? v[i + w] : v[i];
      v[i] = keep + __shfl_xor_sync(kFull, send, 1 << s);
    }
  }
  float r = v[0];
#pragma unroll
  for (int m = NV; m < 32; m <<= 1) r += __shfl_xor_sync(kFull, r, m);
  return r;
}

template <int NV>
__device__ __forceinline__ int transpose_index(int lane) {
  int idx = 0;
#pragma unroll
  for (int s = 0; s < ilog2(NV); ++s) idx += ((lane >> s) & 1) * (NV >> (s + 1));
  return idx;
}

// Rotate-half pairs (group c, group c + HC) of the lane layout, c < HC.
template <int NC, int HC>
__device__ __forceinline__ void rope_groups(float (&x)[NC][4], int lane, const float4* t) {
#pragma unroll
  for (int c = 0; c < HC; ++c) {
    const float4 a = t[2 * lane + 64 * c], b = t[2 * lane + 64 * c + 1];
    const float cs[4] = {a.x, a.z, b.x, b.z}, sn[4] = {a.y, a.w, b.y, b.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float u = x[c][e], w = x[c + HC][e];
      x[c][e] = u * cs[e] - w * sn[e];
      x[c + HC][e] = w * cs[e] + u * sn[e];
    }
  }
}

// RoPE on a row held in the lane layout (x[c][e] = dim 4 lane + 128 c + e),
// given its position's row of the (cos, sin) table (shared or global memory).
template <int NC>
__device__ __forceinline__ void rope_lane(float (&x)[NC][4], int lane, const float4* t, const LayerArgs& la) {
  const int half = la.rot >> 1;
  if (half >= 128) {
    // half the rotated slice is 1 or 2 whole groups per lane
    if (NC == 4 && half == 256)
      rope_groups<NC, NC / 2>(x, lane, t);
    else
      rope_groups<NC, 1>(x, lane, t);
  } else if (half > 0) {
    // rotated slice inside the first 128 dims: lane l < R/4 holds rotated
    // dims, its partner dims are in lane l ^ (half/4)
    const int q = half >> 2;
    float pr[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) pr[e] = __shfl_xor_sync(kFull, x[0][e], q);
    if (4 * lane < la.rot) {
      const float4 a = t[2 * (lane & (q - 1))], b = t[2 * (lane & (q - 1)) + 1];
      const float cs[4] = {a.x, a.z, b.x, b.z}, sn[4] = {a.y, a.w, b.y, b.w};
      const float sg = (lane & q) ? 1.f : -1.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) x[0][e] = x[0][e] * cs[e] + sg * pr[e] * sn[e];
    }
  }
}

// ---- the same, on pairs of dims (x[c][i] = dims 4 lane + 128 c + 2i, +1), with
// the packed two-wide fp32 instructions of sm_100
__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

template <int NC>
__device__ __forceinline__ void load_lane2(const uint8_t* row, int lane, float2 (&x)[NC][2]) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + 8 * lane + 256 * c);
    x[c][0] = unpack_bf16x2(u.x);
    x[c][1] = unpack_bf16x2(u.y);
  }
}

// the same from an int8 row (x[c][i] = codes of dims 4 lane + 128 c + 2i, +1)
template <int NC>
__device__ __forceinline__ void load_lane_q8(const uint8_t* row, int lane, float2 (&x)[NC][2]) {
#pragma unroll
  for (int c = 0; c < NC; ++c)
    unpack_i8x4(*reinterpret_cast<const uint32_t*>(row + 4 * lane + 128 * c), x[c][0], x[c][1]);
}

template <int NC>
__device__ __forceinline__ void zero_lane2(float2 (&x)[NC][2]) {
#pragma unroll
  for (int c = 0; c < NC; ++c) x[c][0] = x[c][1] = f2(0.f, 0.f);
}

// rotate-half pairs (group c, group c + HC), c < HC; t = the position's table row
template <int NC, int HC>
__device__ __forceinline__ void rope_groups2(float2 (&x)[NC][2], int lane, const float4* t) {
#pragma unroll
  for (int c = 0; c < HC; ++c) {
    const float4 a = t[2 * lane + 64 * c], b = t[2 * lane + 64 * c + 1];
    const float2 cs[2] = {f2(a.x, a.z), f2(b.x, b.z)}, sn[2] = {f2(a.y, a.w), f2(b.y, b.w)};
#pragma unroll
    for (int i = 0; i < 2; ++i) {
      const float2 u = x[c][i], w = x[c + HC][i];
      x[c][i] = __ffma2_rn(u, cs[i], __fmul2_rn(f2(-w.x, -w.y), sn[i]));
      x[c + HC][i] = __ffma2_rn(w, cs[i], __fmul2_rn(u, sn[i]));
    }
  }
}

// rotated slice inside the first 128 dims: lanes l < R/4 hold rotated dims,
// the partner dims sit in lane l ^ (R/8); other lanes keep their values
template <int NC>
__device__ __forceinline__ void rope_partner2(float2 (&x)[NC][2], int lane, const float4* t, int rot) {
  const int q = rot >> 3;
  float2 pr[2];
#pragma unroll
  for (int i = 0; i < 2; ++i)
    pr[i] = f2(__shfl_xor_sync(kFull, x[0][i].x, q), __shfl_xor_sync(kFull, x[0][i].y, q));
  const bool in = 4 * lane < rot;
  const int j = in ? 2 * (lane & (q - 1)) : 0;
  const float4 a = t[j], b = t[j + 1];
  const float sg = (lane & q) ? 1.f : -1.f;
  const float2 cs[2] = {f2(a.x, a.z), f2(b.x, b.z)};
  const float2 sn[2] = {f2(sg * a.y, sg * a.w), f2(sg * b.y, sg * b.w)};
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float2 y = __ffma2_rn(x[0][i], cs[i], __fmul2_rn(pr[i], sn[i]));
    x[0][i] = in ? y : x[0][i];
  }
}

template <int NC>
__device__ __forceinline__ void unpack_lane(const uint8_t* row, int lane, float (&x)[NC][4]) {
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    const uint2 u = *reinterpret_cast<const uint2*>(row + 8 * lane + 256 * c);
    const float2 a = unpack_bf16x2(u.x), b = unpack_bf16x2(u.y);
    x[c][0] = a.x;
    x[c][1] = a.y;
    x[c][2] = b.x;
    x[c][3] = b.y;
  }
}

}  // namespace

template <int D, int G, bool KEQV, bool Q8>
__global__ void __launch_bounds__(kSW * 32, 1) decode_simt_kernel(const __grid_constant__ SimtParams P) {
  using C = SimtShape<D, G, KEQV, Q8>;
  constexpr int NC = C::NC, RPW = C::RPW, NV = C::NV;
  const DecodeArgs& da = P.da;
  const LayerArgs& la = P.la;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((128 - (smem_u32(smem_raw) & 127)) & 127);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  int* done_cnt = reinterpret_cast<int*>(full + C::NST);  // [NST] warps done with a stage, cumulative
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::NST; ++s) {
      mbar_init(&full[s], 1);
      done_cnt[s] = 0;
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  const int Hkv = la.Hkv, SUB = kSW / Hkv;
  const int TP = C::ROWS / Hkv;  // positions per tile
  const long long N = static_cast<long long>(da.B) * P.nch;
  const long long i0 = static_cast<long long>(blockIdx.x) * N / gridDim.x;
  const long long i1 = static_cast<long long>(blockIdx.x + 1) * N / gridDim.x;
  if (i1 <= i0) return;  // (never: the grid is at most N)
  const int b_first = static_cast<int>(i0 / P.nch), b_last = static_cast<int>((i1 - 1) / P.nch);
  const uint64_t tmo = P.timeout_ns;
  const size_t row_elems = static_cast<size_t>(Hkv) * D;  // one cache position
  const int half = la.rot >> 1;
  // a cache of transformed keys: no key norm and no key rotation
  const bool knorm = la.qk_norm && !la.kt_cache;
  const int khalf = la.kt_cache ? 0 : half;
  // the (cos, sin) rows of a tile's positions travel with the tile when they fit
  const bool tab_staged = khalf > 0 && TP * half * static_cast<int>(sizeof(float2)) <= kTabBytes;

  // ------------------------------------------------------------ tile copies
  // Stage st of tile u is refilled with tile u + NST by the last warp to finish
  // tile u (one arrival counter per stage); warp 0 issues the first NST tiles.
  // Every warp walks the same cursor, NST tiles ahead of the tile it computes.
  const uint8_t* kbase = Q8 ? reinterpret_cast<const uint8_t*>(da.kq) : reinterpret_cast<const uint8_t*>(da.k);
  const uint8_t* vbase = Q8 ? reinterpret_cast<const uint8_t*>(da.vq) : reinterpret_cast<const uint8_t*>(da.v);
  auto issue = [&](int st, int b, int p0, int npos) {
    const uint32_t bytes = static_cast<uint32_t>(npos * row_elems * C::ES);
    const size_t off = (static_cast<size_t>(b) * da.max_len + p0) * row_elems * C::ES;
    // table rows past the table's end are not copied; their positions are
    // flagged and clamped by the compute loop
    const int trows = tab_staged ? max(0, min(npos, la.rope_max_pos - p0)) : 0;
    const uint32_t tbytes = static_cast<uint32_t>(trows * half * sizeof(float2));
    uint8_t* dst = smem + st * C::STAGE;
    fence_proxy_async_smem();  // this stage's earlier reads come before the copies' writes
    mbar_arrive_expect_tx(&full[st], (KEQV ? bytes : 2 * bytes) + tbytes);
    bulk_load(dst, kbase + off, bytes, &full[st]);
    if (!KEQV) bulk_load(dst + C::KT, vbase + off, bytes, &full[st]);
    if (tbytes) bulk_load(dst + C::OFF_TAB, la.rope_tab + static_cast<size_t>(p0) * half, tbytes, &full[st]);
  };
  const int kvh = warp % Hkv, sub = warp / Hkv;
  // int8 cache: this warp's rows' scales of a tile into its slot st (a row
  // past the tile's positions gets 0), as one commit group per tile
  float* ssc = reinterpret_cast<float*>(smem + C::OFF_SSC) + warp * C::SSC_FLOATS;
  auto copy_scales = [&](int st, int b, int p0, int npos) {
    if constexpr (Q8) {
      const int r = lane % C::RPW, kind = lane / C::RPW;  // kind 0: key scale, 1: value scale
      if (lane < 2 * C::RPW && !(KEQV && kind == 1)) {
        float* dst = ssc + (st * 2 + kind) * C::RPW + r;
        const int pr = sub + r * SUB;
        if (pr < npos)
          cp_async4(dst, (kind ? da.vs : da.ks) + (static_cast<size_t>(b) * da.max_len + p0 + pr) * Hkv + kvh);
        else
          *dst = 0.f;
      }
      cp_async_commit();
    }
  };
  TileCursor ahead;
  ahead.init(P, i0, i1, TP);
  {
    int tb, tp0, tn, u = 0;
    for (; u < C::NST && ahead.next(P, &tb, &tp0, &tn); ++u) {
      if (warp == 0 && lane == 0) issue(u, tb, tp0, tn);
      copy_scales(u, tb, tp0, tn);
    }
    if constexpr (Q8)
      for (; u < C::NST; ++u) cp_async_commit();  // NST groups ahead, some empty
  }

  // -------------------------------------------------------------- compute
  auto load_row = [&](const uint8_t* row, float2 (&x)[NC][2]) {
    if constexpr (Q8) load_lane_q8<NC>(row, lane, x);
    else load_lane2<NC>(row, lane, x);
  };
  const int idx = transpose_index<NV>(lane);
  const int ih = idx % G, ir = idx / G;  // this lane's (row, head) after the butterfly
  float* scr = reinterpret_cast<float*>(smem + C::OFF_SCR) + warp * C::SCR_FLOATS;
  const bool cap = la.softcap > 0.f;
  const float qmul = cap ? la.scale / la.softcap : la.scale_log2;
  const float cap_l2 = cap ? la.softcap * 1.4426950408889634f : 0.f;
  const float goff = la.qk_norm == 1 ? 1.f : 0.f;
  float gk[NC][4];  // key gain per owned dim
#pragma unroll
  for (int c = 0; c < NC; ++c) {
    float4 g = make_float4(1.f, 1.f, 1.f, 1.f);
    if (la.qk_norm) {
      g = __ldg(reinterpret_cast<const float4*>(la.k_norm_w) + lane + 32 * c);
      g.x += goff; g.y += goff; g.z += goff; g.w += goff;
    }
    gk[c][0] = g.x; gk[c][1] = g.y; gk[c][2] = g.z; gk[c][3] = g.w;
  }
  // lane holding the tile maximum of head h after the row reduction
  auto head_lane = [&](int h) {
    int src = 0;
#pragma unroll
    for (int k = 0; k < C::LOGG; ++k) src |= ((h >> k) & 1) << (C::LOGNV - 1 - k);
    return src;
  };
  bool ok = true;
  int t = 0;
  for (int b = b_first; b <= b_last && ok; ++b) {
    const Seg sg = segment(P, b, i0, i1);
    const size_t hrow0 = static_cast<size_t>(b) * la.H + static_cast<size_t>(kvh) * G;  // first query head
    auto write_empty = [&](int c) {
      if (lane < G) {
        float* ml = da.part_ml + ((hrow0 + lane) * da.nsplit + c * SUB + sub) * 2;
        ml[0] = -INFINITY;
        ml[1] = 0.f;
      }
    };
    if (sg.bad_len && sg.c0 == 0 && warp == 0 && lane == 0) flag_status(da.status, kStatusBounds);
    for (int c = sg.c0 + 1; c <= sg.c1; ++c) write_empty(c);
    if (sg.ps >= sg.pe) {
      write_empty(sg.c0);
      continue;
    }

    // query rows of this kv head's group: QK-norm, RoPE at position L-1, scale
    float q[G][NC][4];
#pragma unroll
    for (int h = 0; h < G; ++h) unpack_lane<NC>(reinterpret_cast<const uint8_t*>(da.q + (hrow0 + h) * D), lane, q[h]);
    const int qpos = la.rot > 0 ? checked_pos(sg.L - 1, la, da.status) : 0;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      if (la.qk_norm) {
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int e = 0; e < 4; ++e) ss = fmaf(q[h][c][e], q[h][c][e], ss);
        const float rq = rsqrtf(warp_sum(ss) / static_cast<float>(D) + la.eps);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float4 g = __ldg(reinterpret_cast<const float4*>(la.q_norm_w) + lane + 32 * c);
          q[h][c][0] *= rq * (g.x + goff); q[h][c][1] *= rq * (g.y + goff);
          q[h][c][2] *= rq * (g.z + goff); q[h][c][3] *= rq * (g.w + goff);
        }
      }
      if (la.rot > 0)
        rope_lane<NC>(q[h], lane, reinterpret_cast<const float4*>(la.rope_tab + static_cast<size_t>(qpos) * half), la);
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) q[h][c][e] *= qmul;
    }

    float2 q2[G][NC][2], o2[G][NC][2];
    float m[G];
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m[h] = -INFINITY;
#pragma unroll
      for (int c = 0; c < NC; ++c) {
        q2[h][c][0] = f2(q[h][c][0], q[h][c][1]);
        q2[h][c][1] = f2(q[h][c][2], q[h][c][3]);
        o2[h][c][0] = o2[h][c][1] = f2(0.f, 0.f);
      }
    }
    float lacc = 0.f;  // running sum of this lane's (row, head) slot

    for (int p0 = sg.ps; p0 < sg.pe; p0 += TP, ++t) {
      const int st = t % C::NST;
      if (!__all_sync(kFull, mbar_wait(&full[st], (t / C::NST) & 1, tmo, da.status, abort_flag))) {
        ok = false;
        break;
      }
      if constexpr (Q8) {
        cp_async_wait<C::NST - 1>();  // this tile's scales (group t) have landed
        __syncwarp();
      }
      const float* sk = ssc + st * 2 * C::RPW;    // Q8: key scales of this warp's rows
      const float* sv = KEQV ? sk : sk + C::RPW;  // and value scales
      const uint8_t* kt = smem + st * C::STAGE;
      const uint8_t* vt = KEQV ? kt : kt + C::KT;
      const bool full_tile = p0 + TP <= sg.pe;
      auto row_ptr = [&](const uint8_t* base, int r) {
        return base + static_cast<size_t>((sub + r * SUB) * Hkv + kvh) * D * C::ES;
      };
      // ---- logits of this warp's rows, RB rows at a time.  Each step runs
      // over the RB rows before the next starts (loads, norms, rotation,
      // dots), with no branch inside a step on full tiles, so that the rows'
      // instructions interleave.
      constexpr int RB = RPW;
      float part[NV], ssr[RPW];
      const bool staged = tab_staged && p0 + TP <= la.rope_max_pos;
#pragma unroll
      for (int r0 = 0; r0 < RPW; r0 += RB) {
        float2 k2[RB][NC][2];
        if (full_tile) {
#pragma unroll
          for (int r = 0; r < RB; ++r) load_row(row_ptr(kt, r0 + r), k2[r]);
        } else {
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            if (p0 + sub + (r0 + r) * SUB < sg.pe) load_row(row_ptr(kt, r0 + r), k2[r]);
            else zero_lane2<NC>(k2[r]);
          }
        }
        if (knorm) {
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            float2 a2 = __fmul2_rn(k2[r][0][0], k2[r][0][0]);
            a2 = __ffma2_rn(k2[r][0][1], k2[r][0][1], a2);
#pragma unroll
            for (int c = 1; c < NC; ++c) {
              a2 = __ffma2_rn(k2[r][c][0], k2[r][c][0], a2);
              a2 = __ffma2_rn(k2[r][c][1], k2[r][c][1], a2);
            }
            ssr[r0 + r] = a2.x + a2.y;
#pragma unroll
            for (int c = 0; c < NC; ++c) {
              k2[r][c][0] = __fmul2_rn(k2[r][c][0], f2(gk[c][0], gk[c][1]));
              k2[r][c][1] = __fmul2_rn(k2[r][c][1], f2(gk[c][2], gk[c][3]));
            }
          }
        }
        if (khalf > 0) {
          // the position's table row: staged with the tile (shared-memory
          // loads), else from global memory (positions past the table flagged
          // and clamped); two separate loops so that each load has one space
          const int rk = (NC == 4 && half == 256) ? 2 : half >= 128 ? 1 : 0;
          auto rope_rows = [&](auto kind, auto table_row) {
            constexpr int K = decltype(kind)::value;
#pragma unroll
            for (int r = 0; r < RB; ++r) {
              const float4* tr = table_row(r0 + r);
              if constexpr (K == 2) rope_groups2<NC, NC / 2>(k2[r], lane, tr);
              else if constexpr (K == 1) rope_groups2<NC, 1>(k2[r], lane, tr);
              else rope_partner2<NC>(k2[r], lane, tr, la.rot);
            }
          };
          auto rope_all = [&](auto table_row) {
            if (rk == 2) rope_rows(std::integral_constant<int, 2>{}, table_row);
            else if (rk == 1) rope_rows(std::integral_constant<int, 1>{}, table_row);
            else rope_rows(std::integral_constant<int, 0>{}, table_row);
          };
          if (staged) {
            const uint8_t* tb = kt + C::OFF_TAB + static_cast<size_t>(sub) * half * 8;
            rope_all([&](int r) {
              return reinterpret_cast<const float4*>(tb + static_cast<size_t>(r * SUB) * half * 8);
            });
          } else {
            rope_all([&](int r) {
              const int pos = min(p0 + sub + r * SUB, sg.pe - 1);
              return reinterpret_cast<const float4*>(la.rope_tab +
                                                     static_cast<size_t>(checked_pos(pos, la, da.status)) * half);
            });
          }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
          for (int h = 0; h < G; ++h) {
            float2 a2 = __fmul2_rn(q2[h][0][0], k2[r][0][0]);
            a2 = __ffma2_rn(q2[h][0][1], k2[r][0][1], a2);
#pragma unroll
            for (int c = 1; c < NC; ++c) {
              a2 = __ffma2_rn(q2[h][c][0], k2[r][c][0], a2);
              a2 = __ffma2_rn(q2[h][c][1], k2[r][c][1], a2);
            }
            part[(r0 + r) * G + h] = a2.x + a2.y;
          }
      }
      float x = transpose_sum<NV>(part, lane);
      if (knorm) {
        // 1/rms of each row: sums of squares through the same butterfly, then
        // each row's factor from the warp scratch
        float s2 = transpose_sum<RPW>(ssr, lane);
        const int ri = transpose_index<RPW>(lane);
        if constexpr (Q8) s2 *= sk[ri] * sk[ri];  // of the dequantised row
        __syncwarp();
        scr[32 + ri] = rsqrtf(s2 / static_cast<float>(D) + la.eps);
        __syncwarp();
        x *= scr[32 + ir];
      }
      if constexpr (Q8) x *= sk[ir];
      const bool vis = p0 + sub + ir * SUB < sg.pe;
      x = vis ? (cap ? cap_l2 * tanh_fast(x) : x) : -INFINITY;
      // ---- online softmax: tile maxima per head (over the row bits of idx)
      float mx = x;
#pragma unroll
      for (int k = 0; k < C::LOGNV - C::LOGG; ++k) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1 << k));
      float alpha[G], mnew_own = 0.f, alpha_own = 1.f;
      bool rescale = false;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mt = __shfl_sync(kFull, mx, head_lane(h));
        const float mn = fmaxf(m[h], mt);
        alpha[h] = (m[h] == -INFINITY) ? 0.f : ex2(m[h] - mn);
        rescale = rescale || (mn != m[h]);
        m[h] = mn;
        if (h == ih) {
          mnew_own = mn;
          alpha_own = alpha[h];
        }
      }
      const float p = vis ? ex2(x - mnew_own) : 0.f;
      lacc = lacc * alpha_own + p;
      __syncwarp();
      scr[idx] = Q8 ? p * sv[ir] : p;  // P V reads the value scale with the weight
      __syncwarp();
      float pv[NV];
#pragma unroll
      for (int i = 0; i < NV; i += 4) {
        const float4 f = *reinterpret_cast<const float4*>(scr + i);
        pv[i] = f.x; pv[i + 1] = f.y; pv[i + 2] = f.z; pv[i + 3] = f.w;
      }
      if (rescale) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            o2[h][c][0] = __fmul2_rn(o2[h][c][0], f2(alpha[h], alpha[h]));
            o2[h][c][1] = __fmul2_rn(o2[h][c][1], f2(alpha[h], alpha[h]));
          }
      }
      // ---- P V, RB rows at a time (rows past the segment are zero: p = 0 times 0)
#pragma unroll
      for (int r0 = 0; r0 < RPW; r0 += RB) {
        float2 v2[RB][NC][2];
        if (full_tile) {
#pragma unroll
          for (int r = 0; r < RB; ++r) load_row(row_ptr(vt, r0 + r), v2[r]);
        } else {
#pragma unroll
          for (int r = 0; r < RB; ++r) {
            if (p0 + sub + (r0 + r) * SUB < sg.pe) load_row(row_ptr(vt, r0 + r), v2[r]);
            else zero_lane2<NC>(v2[r]);
          }
        }
#pragma unroll
        for (int r = 0; r < RB; ++r)
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float2 pp = f2(pv[(r0 + r) * G + h], pv[(r0 + r) * G + h]);
#pragma unroll
            for (int c = 0; c < NC; ++c) {
              o2[h][c][0] = __ffma2_rn(v2[r][c][0], pp, o2[h][c][0]);
              o2[h][c][1] = __ffma2_rn(v2[r][c][1], pp, o2[h][c][1]);
            }
          }
      }
      __syncwarp();
      {
        int tb, tp0, tn;
        const bool more = ahead.next(P, &tb, &tp0, &tn);  // tile t + NST, if any
        __threadfence_block();  // this warp's reads of the stage are done
        if (lane == 0 && (atomicAdd(&done_cnt[st], 1) % kSW) == kSW - 1 && more) issue(st, tb, tp0, tn);
        if constexpr (Q8) {
          if (more) copy_scales(st, tb, tp0, tn);
          else cp_async_commit();
        }
      }
    }
    if (!ok) break;
    // ---- this segment's partial: l per head over the row bits, then O and (m, l)
    float ls = lacc;
#pragma unroll
    for (int k = 0; k < C::LOGNV - C::LOGG; ++k) ls += __shfl_xor_sync(kFull, ls, 1 << k);
    const int slot = sg.c0 * SUB + sub;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      const float lh = __shfl_sync(kFull, ls, head_lane(h));
      const size_t prow = (hrow0 + h) * da.nsplit + slot;
      float* dst = da.part_o + prow * D;
#pragma unroll
      for (int c = 0; c < NC; ++c)
        *reinterpret_cast<float4*>(dst + 4 * lane + 128 * c) =
            make_float4(o2[h][c][0].x, o2[h][c][0].y, o2[h][c][1].x, o2[h][c][1].y);
      if (lane == 0) {
        da.part_ml[prow * 2] = m[h];
        da.part_ml[prow * 2 + 1] = lh;
      }
    }
  }
  if constexpr (Q8) cp_async_wait<0>();  // no scale copy outlives the CTA
  if (*abort_flag) {
    // after a failed wait, copies issued just before it may still be landing:
    // give them ~100 us before the CTA may exit
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 100000) {
    }
  }
}

namespace {

// SM count of the current device, queried once per device (148 if the query fails).
int device_sm_count() {
  constexpr int kMaxDev = 64;
  static int sms[kMaxDev] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDev) return 148;
  if (sms[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    sms[dev] = n;
  }
  return sms[dev];
}

template <int D, int G, bool KEQV, bool Q8>
cudaError_t run_decode_simt(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  using C = SimtShape<D, G, KEQV, Q8>;
  constexpr int kMaxDev = 64;
  static bool attr_set[kMaxDev] = {};
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  auto kern = decode_simt_kernel<D, G, KEQV, Q8>;
  if (!attr_set[dev]) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set[dev] = true;
  }
  SimtParams P;
  P.da = da;
  P.la = la;
  P.nch = da.nsplit / (kSW / la.Hkv);
  P.timeout_ns = wait_timeout_ns();
  const long long items = static_cast<long long>(da.B) * P.nch;
  if (items <= 0) return cudaSuccess;
  const long long grid = items < sms ? items : sms;
  kern<<<static_cast<unsigned>(grid), kSW * 32, C::SMEM, s>>>(P);
  return cudaGetLastError();
}

}  // namespace

bool decode_simt_supported(const LayerArgs& la) {
  if (la.Hkv != 1 && la.Hkv != 2 && la.Hkv != 4 && la.Hkv != 8) return false;
  if (la.D == 256) return la.G == 1 || la.G == 2 || la.G == 4;
  if (la.D == 512) return la.G == 1 || la.G == 2;
  return false;
}

// Chunks per sequence: about 16 work items per SM over the batch (so that
// equal ranges of items balance), at least one tile per chunk, at most 64
// chunks and at most max_split split slots.
void decode_simt_plan(const LayerArgs& la, int B, int max_len, int max_split, int* nsplit, int* chunk) {
  const int SUB = kSW / la.Hkv;
  const int TP = kTileBytes / (2 * la.D) / la.Hkv;
  const int span = la.window > 0 ? (la.window < max_len ? la.window : max_len) : max_len;
  const int sms = device_sm_count();
  int nch = (16 * sms + (B > 0 ? B : 1) - 1) / (B > 0 ? B : 1);
  const int tiles = (span + TP - 1) / TP;
  if (nch > tiles) nch = tiles;
  if (nch > 64) nch = 64;
  if (nch > max_split / SUB) nch = max_split / SUB;
  if (nch < 1) nch = 1;
  const int c = (span + nch - 1) / nch;
  *chunk = c;
  *nsplit = ((span + c - 1) / c) * SUB;
}

template <bool Q8>
static cudaError_t launch_decode_simt_t(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  if (la.D == 256) {
    if (la.k_eq_v) {
      switch (la.G) {
        case 1: return run_decode_simt<256, 1, true, Q8>(da, la, s);
        case 2: return run_decode_simt<256, 2, true, Q8>(da, la, s);
        case 4: return run_decode_simt<256, 4, true, Q8>(da, la, s);
      }
    } else {
      switch (la.G) {
        case 1: return run_decode_simt<256, 1, false, Q8>(da, la, s);
        case 2: return run_decode_simt<256, 2, false, Q8>(da, la, s);
        case 4: return run_decode_simt<256, 4, false, Q8>(da, la, s);
      }
    }
  } else if (la.D == 512) {
    if (la.k_eq_v) {
      switch (la.G) {
        case 1: return run_decode_simt<512, 1, true, Q8>(da, la, s);
        case 2: return run_decode_simt<512, 2, true, Q8>(da, la, s);
      }
    } else {
      switch (la.G) {
        case 1: return run_decode_simt<512, 1, false, Q8>(da, la, s);
        case 2: return run_decode_simt<512, 2, false, Q8>(da, la, s);
      }
    }
  }
  return cudaErrorInvalidValue;
}

// an int8 cache when da.kq is set, else bf16
cudaError_t launch_decode_simt(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s) {
  return da.kq ? launch_decode_simt_t<true>(da, la, s) : launch_decode_simt_t<false>(da, la, s);
}

}  // namespace gattn
