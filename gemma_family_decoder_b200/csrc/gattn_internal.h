// Internal launcher interface between the C-ABI host code (gattn_api.cu) and
// the kernel translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gattn.h"

namespace gattn {

// Fields shared by every kernel, resolved from gattn_cfg on the host.
struct LayerArgs {
  int H, Hkv, G, D;
  int window;
  int rot;             // rotated dims R (0, or a power of two multiple of 16, <= D)
  int rope_max_pos;
  const float2* rope_tab;  // [max_pos][R/2] (cos, sin)
  double rope_ratio;      // theta^(-2/F): pair t turns theta^(-2t/F) = rope_ratio^t per position
  float softcap;       // 0 = off
  float scale_log2;    // scalar^-1/2 * log2(e)
  float scale;         // scalar^-1/2
  int qk_norm;         // 0 none, 1 (1+w), 2 w
  float eps;
  const float* q_norm_w;
  const float* k_norm_w;
  int k_eq_v;
  int kt_cache;        // caches hold transformed keys: decode kernels skip the key norm and RoPE
};

// RoPE table: (cos, sin) of p * theta^(-2t/F) for p < max_pos, t < half.
cudaError_t launch_rope_table(float2* tab, double theta, int half, int freq_dim, int max_pos,
                              cudaStream_t s);

// The chunk form of launch_qkprep (below): queries of a chunk (token prefix[b] + i,
// q only) into qt, and cache keys (token j, rows j < prefix[b] + C only) into kt.
cudaError_t launch_qkprep_chunk(const __nv_bfloat16* q, const __nv_bfloat16* k_cache, const int* prefix,
                                __nv_bfloat16* qt, __nv_bfloat16* kt, int B, int C, int max_len,
                                const LayerArgs& la, uint32_t* status, cudaStream_t s, bool with_keys);
// Copy a chunk's new rows [B][C][Hkv][D] into cache rows [prefix[b], prefix[b] + C)
// (v_new / v_cache null when keys and values are tied); a prefix outside
// [0, max_len - C] is clamped and flagged.
cudaError_t launch_kv_append(const __nv_bfloat16* k_new, const __nv_bfloat16* v_new, __nv_bfloat16* k_cache,
                             __nv_bfloat16* v_cache, const int* prefix, int B, int C, int max_len, int Hkv,
                             int D, uint32_t* status, cudaStream_t s);
// A chunk's new keys [B][C][Hkv][D] transformed at positions prefix[b] + s and
// written to cache rows prefix[b] + s (a transformed cache's append).
cudaError_t launch_key_append_transformed(const __nv_bfloat16* k_new, __nv_bfloat16* k_cache, const int* prefix,
                                          int B, int C, int max_len, const LayerArgs& la, uint32_t* status,
                                          cudaStream_t s);
// q~ = RoPE(RMSNorm(q)) for every (b, s, head) row and k~ = RoPE(RMSNorm(k))
// for every (b, s, kv head) row, bf16 out, same layouts, in one launch.
cudaError_t launch_qkprep(const __nv_bfloat16* q, const __nv_bfloat16* k, const int* positions,
                          __nv_bfloat16* qt, __nv_bfloat16* kt, int B, int S, const LayerArgs& la,
                          uint32_t* status, cudaStream_t s);

// Split-KV decode: partials (m, l, O) per (b, h, split) then the merge.
struct DecodeArgs {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const int* seq_lens;
  __nv_bfloat16* out;
  int B, max_len;
  int nsplit, chunk;
  float* part_o;   // [B][H][nsplit][D]
  float* part_ml;  // [B][H][nsplit][2]
  uint32_t* status;
  unsigned long long* trace = nullptr;  // optional per-CTA timeline (tensor-core kernel)
  size_t trace_bytes = 0;
  // int8 cache (instead of k / v): codes [B][max_len][Hkv][D], fp32 scales [B][max_len][Hkv]
  const int8_t* kq = nullptr;
  const int8_t* vq = nullptr;
  const float* ks = nullptr;
  const float* vs = nullptr;
};
// Split plan of a decode call: keys per chunk and split slots per (b, head),
// with at most `max_split` slots (fewer, longer chunks when the plan would
// exceed it; callers check the result against their own limit).
void decode_plan(const LayerArgs& la, int B, int max_len, int* nsplit, int* chunk,
                 int max_split = 1 << 30);
// Partials of every split, by the kernel that fits the layer, then nothing else
// (the merge is launch_decode_combine).
cudaError_t launch_decode_split(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s);
cudaError_t launch_decode_combine(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s);
// Tensor-core split kernel: K=V layers with 8 or 16 query heads per kv head,
// head_dim 256 or 512 and at most 128 rotated dims, bf16 or int8 caches (same
// partial format).
bool decode_tc_supported(const LayerArgs& la);
cudaError_t launch_decode_tc(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s);
// Persistent CUDA-core split kernel for 1, 2 or 4 query heads per kv head
// (head_dim 512: 1 or 2) and 1, 2, 4 or 8 kv heads; its own plan.
bool decode_simt_supported(const LayerArgs& la);
void decode_simt_plan(const LayerArgs& la, int B, int max_len, int max_split, int* nsplit, int* chunk);
cudaError_t launch_decode_simt(const DecodeArgs& da, const LayerArgs& la, cudaStream_t s);
// int8 cache rows: codes and scales of nrows rows of head_dim D (256 or 512)
cudaError_t launch_kv_quantize(const __nv_bfloat16* x, int8_t* codes, float* scales, long long nrows, int D,
                               cudaStream_t s);

// Prefill on tcgen05 tensor cores.
struct PrefillArgs {
  const __nv_bfloat16* q;   // transformed queries (or raw q when no transform applies)
  const __nv_bfloat16* kt;  // transformed keys (or raw k when no transform applies)
  const __nv_bfloat16* v;   // values (raw k when k_eq_v)
  __nv_bfloat16* out;
  int B, S;
  uint32_t* status;
  uint64_t timeout_ns;
  unsigned long long* trace;  // optional kernel timeline buffer (null = off)
  size_t trace_bytes;
  const int* seq_range = nullptr;  // [B][2] valid tokens of each sequence (padded batch), or null
  // a chunk against a cached prefix: query row i of sequence b is token q_off[b] + i; the
  // keys and values have KV_S rows (the cache), q and out S rows
  const int* q_off = nullptr;
  int KV_S = 0;
};
cudaError_t launch_prefill(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s);

// Head_dim 512 prefill on SM pairs (tcgen05 cta_group::2; see
// prefill_pair.cu): whole prompts of layers with an even number of query heads
// per kv head.  Same arguments as launch_prefill.
bool prefill_pair_supported(const LayerArgs& la);
cudaError_t launch_prefill_pair(const PrefillArgs& pa, const LayerArgs& la, cudaStream_t s);

// Self-test: one CTA waits on an mbarrier nobody arrives on.
cudaError_t launch_selftest_wait(uint32_t* status, uint64_t timeout_ns, cudaStream_t s);

// Host checks of a decode call without its workspace arguments (the same
// checks gattn_decode makes); fills `la`.  Returns a gattn_status.
int check_decode_call(const gattn_cfg* cfg, const void* q, const void* k_cache,
                      const void* v_cache_or_null, const int32_t* seq_lens, const void* out,
                      int32_t batch, int32_t max_len, LayerArgs* la);
// Record `msg` as this thread's last error and return `code`.
int report_error(int code, const char* msg);

// Launch `kern` on `s` with programmatic stream serialization: its CTAs may be
// scheduled before the previous kernel in the stream finishes, and must call
// pdl_wait() before reading what that kernel wrote.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

// Wait limit used by every launch (ns).
uint64_t wait_timeout_ns();

// TMA descriptor encoding through the driver entry point (no -lcuda needed).
bool encode_tmap_bshd(CUtensorMap* map, const void* base, int B, int S, int Hkv, int D,
                      int box_rows);
// The same view of an int8 cache [B][S][Hkv][D] (codes), box box_inner bytes x box_rows rows.
bool encode_tmap_bshd_u8(CUtensorMap* map, const void* base, int B, int S, int Hkv, int D, int box_inner,
                         int box_rows);

}  // namespace gattn
