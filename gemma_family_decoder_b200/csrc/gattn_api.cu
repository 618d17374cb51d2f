// C ABI of libgattn: argument checks, workspace layout, kernel choice and
// launches.  Every public function is declared (and documented) in
// include/gattn.h.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "gattn.h"
#include "gattn_internal.h"

namespace {

thread_local char g_last_error[512] = "";
thread_local cudaEvent_t g_prof_start = nullptr;
thread_local cudaEvent_t g_prof_stop = nullptr;
thread_local void* g_trace_buf = nullptr;
thread_local size_t g_trace_bytes = 0;
uint64_t g_timeout_ns = 2000000ull * 1000ull;  // 2 s

int fail(int code, const char* fmt, const char* detail = nullptr) {
  if (detail)
    std::snprintf(g_last_error, sizeof(g_last_error), fmt, detail);
  else
    std::snprintf(g_last_error, sizeof(g_last_error), "%s", fmt);
  return code;
}

int fail_cuda(cudaError_t e, const char* where) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s: %s", where, cudaGetErrorString(e));
  return GATTN_ERR_CUDA;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kStatusBytes = 256;

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Resolve and check a gattn_cfg.  `need_rope_ptr` is false for pure size queries.
int resolve(const gattn_cfg* cfg, gattn::LayerArgs* la, bool need_ptrs) {
  if (!cfg) return fail(GATTN_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->num_heads <= 0 || cfg->num_kv_heads <= 0)
    return fail(GATTN_ERR_INVALID_ARG, "num_heads and num_kv_heads must be positive");
  if (cfg->num_heads % cfg->num_kv_heads != 0)
    return fail(GATTN_ERR_INVALID_ARG, "num_heads must be a multiple of num_kv_heads");
  if (cfg->head_dim != 256 && cfg->head_dim != 512)
    return fail(GATTN_ERR_UNSUPPORTED, "head_dim must be 256 or 512");
  if (cfg->window < 0) return fail(GATTN_ERR_INVALID_ARG, "window must be >= 0");
  if (!(cfg->rotary_fraction >= 0.f && cfg->rotary_fraction <= 1.f))
    return fail(GATTN_ERR_INVALID_ARG, "rotary_fraction must be in [0, 1]");
  const int D = cfg->head_dim;
  const float rf = cfg->rotary_fraction * static_cast<float>(D);
  const int R = static_cast<int>(std::lround(rf));
  if (std::fabs(rf - static_cast<float>(R)) > 1e-3f)
    return fail(GATTN_ERR_INVALID_ARG, "rotary_fraction * head_dim must be an integer");
  if (R != 0 && R != 16 && R != 32 && R != 64 && R != 128 && R != 256 && R != 512)
    return fail(GATTN_ERR_UNSUPPORTED, "rotated dims must be 0 or a power of two in [16, 512]");
  if (R > D) return fail(GATTN_ERR_INVALID_ARG, "rotated dims exceed head_dim");
  if (R > 0 && need_ptrs) {
    if (!cfg->rope_table) return fail(GATTN_ERR_INVALID_ARG, "rope_table is NULL with RoPE on");
    if (!aligned16(cfg->rope_table)) return fail(GATTN_ERR_INVALID_ARG, "rope_table misaligned");
    if (cfg->rope_max_pos <= 0) return fail(GATTN_ERR_INVALID_ARG, "rope_max_pos must be > 0");
  }
  if (cfg->rope_freq_dim < 0) return fail(GATTN_ERR_INVALID_ARG, "rope_freq_dim must be >= 0");
  if (!(cfg->softcap >= 0.f) || std::isinf(cfg->softcap))
    return fail(GATTN_ERR_INVALID_ARG, "softcap must be finite and >= 0");
  if (!(cfg->scalar > 0.f) || std::isinf(cfg->scalar))
    return fail(GATTN_ERR_INVALID_ARG, "scalar must be finite and > 0");
  if (cfg->k_eq_v != 0 && cfg->k_eq_v != 1) return fail(GATTN_ERR_INVALID_ARG, "k_eq_v must be 0 or 1");
  if (cfg->keys_transformed != 0 && cfg->keys_transformed != 1)
    return fail(GATTN_ERR_INVALID_ARG, "keys_transformed must be 0 or 1");
  if (cfg->keys_transformed && cfg->k_eq_v)
    return fail(GATTN_ERR_INVALID_ARG, "keys_transformed with k_eq_v: tied values need the raw keys");
  if (cfg->qk_norm < 0 || cfg->qk_norm > 2) return fail(GATTN_ERR_INVALID_ARG, "qk_norm must be 0, 1 or 2");
  if (cfg->qk_norm != 0) {
    if (!(cfg->norm_eps >= 0.f)) return fail(GATTN_ERR_INVALID_ARG, "norm_eps must be >= 0");
    if (need_ptrs && (!cfg->q_norm_w || !cfg->k_norm_w))
      return fail(GATTN_ERR_INVALID_ARG, "QK-norm weights are NULL with qk_norm on");
    if (need_ptrs && (!aligned16(cfg->q_norm_w) || !aligned16(cfg->k_norm_w)))
      return fail(GATTN_ERR_INVALID_ARG, "QK-norm weights must be 16-byte aligned");
  }
  la->H = cfg->num_heads;
  la->Hkv = cfg->num_kv_heads;
  la->G = cfg->num_heads / cfg->num_kv_heads;
  la->D = D;
  la->window = cfg->window;
  la->rot = R;
  la->rope_max_pos = cfg->rope_max_pos;
  la->rope_tab = reinterpret_cast<const float2*>(cfg->rope_table);
  la->rope_ratio = std::pow(static_cast<double>(cfg->rope_theta),
                            -2.0 / static_cast<double>(cfg->rope_freq_dim ? cfg->rope_freq_dim : D));
  la->softcap = cfg->softcap;
  la->scale = 1.0f / std::sqrt(cfg->scalar);
  la->scale_log2 = la->scale * 1.4426950408889634f;
  la->qk_norm = cfg->qk_norm;
  la->eps = cfg->norm_eps;
  la->q_norm_w = cfg->q_norm_w;
  la->k_norm_w = cfg->k_norm_w;
  la->k_eq_v = cfg->k_eq_v;
  la->kt_cache = cfg->keys_transformed;
  return GATTN_OK;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

namespace gattn {

uint64_t wait_timeout_ns() { return g_timeout_ns; }

int report_error(int code, const char* msg) { return fail(code, msg); }

int check_decode_call(const gattn_cfg* cfg, const void* q, const void* k_cache,
                      const void* v_cache_or_null, const int32_t* seq_lens, const void* out,
                      int32_t batch, int32_t max_len, LayerArgs* la) {
  g_last_error[0] = 0;
  int st = resolve(cfg, la, true);
  if (st != GATTN_OK) return st;
  const int G = la->G;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
    return fail(GATTN_ERR_UNSUPPORTED, "decode supports num_heads / num_kv_heads in {1,2,4,8,16}");
  if (batch < 0 || max_len <= 0) return fail(GATTN_ERR_INVALID_ARG, "batch must be >= 0 and max_len > 0");
  if (!q || !k_cache || !out || !seq_lens)
    return fail(GATTN_ERR_INVALID_ARG, "q, k_cache, seq_lens and out must not be NULL");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(out))
    return fail(GATTN_ERR_INVALID_ARG, "q, k_cache and out must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(seq_lens) & 3u)
    return fail(GATTN_ERR_INVALID_ARG, "seq_lens must be 4-byte aligned");
  if (la->k_eq_v) {
    if (v_cache_or_null && v_cache_or_null != k_cache)
      return fail(GATTN_ERR_INVALID_ARG, "k_eq_v: v_cache must be NULL or k_cache");
  } else {
    if (!v_cache_or_null) return fail(GATTN_ERR_INVALID_ARG, "v_cache is NULL without k_eq_v");
    if (!aligned16(v_cache_or_null)) return fail(GATTN_ERR_INVALID_ARG, "v_cache must be 16-byte aligned");
  }
  return GATTN_OK;
}

bool encode_tmap_bshd(CUtensorMap* map, const void* base, int B, int S, int Hkv, int D,
                      int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(Hkv) * D * 2,
                                 static_cast<cuuint64_t>(S) * Hkv * D * 2};
  const cuuint32_t box[4] = {64, 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The same 4-D view of an int8 (code) cache: box `box_inner` bytes x box_rows rows.
bool encode_tmap_bshd_u8(CUtensorMap* map, const void* base, int B, int S, int Hkv, int D, int box_inner,
                         int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv),
                              static_cast<cuuint64_t>(S), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Hkv) * D,
                                 static_cast<cuuint64_t>(S) * Hkv * D};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(box_inner), 1, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gattn

extern "C" {

const char* gattn_version(void) { return "libgattn 0.1 sm_100a"; }

const char* gattn_status_string(int s) {
  switch (s) {
    case GATTN_OK: return "ok";
    case GATTN_ERR_INVALID_ARG: return "invalid argument";
    case GATTN_ERR_UNSUPPORTED: return "unsupported configuration";
    case GATTN_ERR_WORKSPACE: return "workspace missing or too small";
    case GATTN_ERR_CUDA: return "CUDA error";
    case GATTN_ERR_TIMEOUT: return "device wait timed out";
    case GATTN_ERR_DEVICE_BOUNDS: return "device index out of range";
    default: return "unknown status";
  }
}

const char* gattn_last_error(void) { return g_last_error; }

int gattn_cp_blocks(int32_t seq_len, int32_t world, int32_t rank, int32_t* starts, int32_t* lens) {
  g_last_error[0] = 0;
  if (!starts || !lens) return fail(GATTN_ERR_INVALID_ARG, "starts and lens must not be NULL");
  if (world < 1) return fail(GATTN_ERR_INVALID_ARG, "world must be >= 1");
  if (rank < 0 || rank >= world) return fail(GATTN_ERR_INVALID_ARG, "rank must be in [0, world)");
  if (seq_len < 0) return fail(GATTN_ERR_INVALID_ARG, "seq_len must be >= 0");
  const int64_t nb = 2 * static_cast<int64_t>(world);
  const int64_t base = seq_len / nb, extra = seq_len % nb;
  // block i: base tokens, one more for the first `extra` blocks
  auto start_of = [&](int64_t i) { return i * base + (i < extra ? i : extra); };
  auto len_of = [&](int64_t i) { return base + (i < extra ? 1 : 0); };
  const int64_t b0 = rank, b1 = nb - 1 - rank;
  starts[0] = static_cast<int32_t>(start_of(b0));
  lens[0] = static_cast<int32_t>(len_of(b0));
  starts[1] = static_cast<int32_t>(start_of(b1));
  lens[1] = static_cast<int32_t>(len_of(b1));
  return GATTN_OK;
}

void gattn_set_wait_timeout_us(uint32_t timeout_us) {
  g_timeout_ns = (timeout_us ? static_cast<uint64_t>(timeout_us) : 2000000ull) * 1000ull;
}

size_t gattn_rope_table_bytes(int32_t max_pos, int32_t rot_dim) {
  if (max_pos <= 0 || rot_dim <= 0 || (rot_dim & 1)) return 0;
  return static_cast<size_t>(max_pos) * (rot_dim / 2) * 2 * sizeof(float);
}

int gattn_rope_table_fill(float* table, float theta, int32_t rot_dim, int32_t freq_dim,
                          int32_t max_pos, gattn_stream stream) {
  g_last_error[0] = 0;
  if (!table || !aligned16(table)) return fail(GATTN_ERR_INVALID_ARG, "table NULL or misaligned");
  if (!(theta > 0.f) || std::isinf(theta)) return fail(GATTN_ERR_INVALID_ARG, "theta must be > 0");
  if (rot_dim <= 0 || (rot_dim & 1)) return fail(GATTN_ERR_INVALID_ARG, "rot_dim must be even and > 0");
  if (freq_dim <= 0) return fail(GATTN_ERR_INVALID_ARG, "freq_dim must be > 0");
  if (max_pos <= 0) return fail(GATTN_ERR_INVALID_ARG, "max_pos must be > 0");
  cudaError_t e = gattn::launch_rope_table(reinterpret_cast<float2*>(table), theta, rot_dim / 2,
                                           freq_dim, max_pos, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GATTN_OK : fail_cuda(e, "rope table launch");
}

int gattn_workspace_init(void* workspace, size_t ws_bytes, gattn_stream stream) {
  g_last_error[0] = 0;
  if (!workspace || !aligned16(workspace)) return fail(GATTN_ERR_INVALID_ARG, "workspace NULL or misaligned");
  if (ws_bytes < kStatusBytes) return fail(GATTN_ERR_WORKSPACE, "workspace smaller than 256 bytes");
  cudaError_t e = cudaMemsetAsync(workspace, 0, kStatusBytes, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GATTN_OK : fail_cuda(e, "workspace init");
}

// ---- prefill ---------------------------------------------------------------------
static bool prefill_needs_kprep(const gattn::LayerArgs& la) { return la.rot > 0 || la.qk_norm != 0; }

size_t gattn_prefill_workspace_size(const gattn_cfg* cfg, int32_t batch, int32_t seq_len) {
  gattn::LayerArgs la;
  if (resolve(cfg, &la, false) != GATTN_OK || batch < 0 || seq_len < 0) return 0;
  size_t bytes = kStatusBytes;
  if (prefill_needs_kprep(la))  // transformed keys, then transformed queries
    bytes = round_up(bytes, 1024) +
            round_up(static_cast<size_t>(batch) * seq_len * la.Hkv * la.D * sizeof(uint16_t), 1024) +
            static_cast<size_t>(batch) * seq_len * la.H * la.D * sizeof(uint16_t);
  return bytes;
}

static int prefill_impl(const gattn_bf16* q, const gattn_bf16* k, const gattn_bf16* v_or_null,
                        const int32_t* positions, const int32_t* seq_range, gattn_bf16* out,
                        int32_t batch, int32_t seq_len, const gattn_cfg* cfg, void* workspace,
                        size_t ws_bytes, gattn_stream stream);

int gattn_prefill(const gattn_bf16* q, const gattn_bf16* k, const gattn_bf16* v_or_null,
                  const int32_t* positions, gattn_bf16* out, int32_t batch, int32_t seq_len,
                  const gattn_cfg* cfg, void* workspace, size_t ws_bytes, gattn_stream stream) {
  g_last_error[0] = 0;
  return prefill_impl(q, k, v_or_null, positions, nullptr, out, batch, seq_len, cfg, workspace, ws_bytes,
                      stream);
}

int gattn_prefill_padded(const gattn_bf16* q, const gattn_bf16* k, const gattn_bf16* v_or_null,
                         const int32_t* positions, const int32_t* seq_range, gattn_bf16* out,
                         int32_t batch, int32_t seq_len, const gattn_cfg* cfg, void* workspace,
                         size_t ws_bytes, gattn_stream stream) {
  g_last_error[0] = 0;
  if (!seq_range) return fail(GATTN_ERR_INVALID_ARG, "seq_range must not be NULL");
  if (reinterpret_cast<uintptr_t>(seq_range) & 3u)
    return fail(GATTN_ERR_INVALID_ARG, "seq_range must be 4-byte aligned");
  return prefill_impl(q, k, v_or_null, positions, seq_range, out, batch, seq_len, cfg, workspace, ws_bytes,
                      stream);
}

static int prefill_impl(const gattn_bf16* q, const gattn_bf16* k, const gattn_bf16* v_or_null,
                        const int32_t* positions, const int32_t* seq_range, gattn_bf16* out,
                        int32_t batch, int32_t seq_len, const gattn_cfg* cfg, void* workspace,
                        size_t ws_bytes, gattn_stream stream) {
  gattn::LayerArgs la;
  int st = resolve(cfg, &la, true);
  if (st != GATTN_OK) return st;
  if (batch < 0 || seq_len < 0) return fail(GATTN_ERR_INVALID_ARG, "batch and seq_len must be >= 0");
  if (static_cast<long long>(seq_len) * batch * la.H > (1LL << 40))
    return fail(GATTN_ERR_INVALID_ARG, "problem too large");
  if (!q || !k || !out) return fail(GATTN_ERR_INVALID_ARG, "q, k and out must not be NULL");
  if (!aligned16(q) || !aligned16(k) || !aligned16(out))
    return fail(GATTN_ERR_INVALID_ARG, "q, k and out must be 16-byte aligned");
  if (la.k_eq_v) {
    if (v_or_null && v_or_null != k) return fail(GATTN_ERR_INVALID_ARG, "k_eq_v: v must be NULL or k");
  } else {
    if (!v_or_null) return fail(GATTN_ERR_INVALID_ARG, "v is NULL without k_eq_v");
    if (!aligned16(v_or_null)) return fail(GATTN_ERR_INVALID_ARG, "v must be 16-byte aligned");
  }
  if (la.rot > 0 && !positions) return fail(GATTN_ERR_INVALID_ARG, "positions NULL with RoPE on");
  if (positions && (reinterpret_cast<uintptr_t>(positions) & 3u))
    return fail(GATTN_ERR_INVALID_ARG, "positions must be 4-byte aligned");
  const size_t need = gattn_prefill_workspace_size(cfg, batch, seq_len);
  if (!workspace || ws_bytes < need) return fail(GATTN_ERR_WORKSPACE, "workspace missing or too small");
  if (!aligned16(workspace)) return fail(GATTN_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (batch == 0 || seq_len == 0) return GATTN_OK;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  const __nv_bfloat16* kb = reinterpret_cast<const __nv_bfloat16*>(k);
  const __nv_bfloat16* kt = kb;
  const __nv_bfloat16* qt = reinterpret_cast<const __nv_bfloat16*>(q);
  const bool prep = prefill_needs_kprep(la);
  if (prep) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    __nv_bfloat16* ktw = reinterpret_cast<__nv_bfloat16*>(ws + round_up(kStatusBytes, 1024));
    __nv_bfloat16* qtw = reinterpret_cast<__nv_bfloat16*>(
        ws + round_up(kStatusBytes, 1024) +
        round_up(static_cast<size_t>(batch) * seq_len * la.Hkv * la.D * sizeof(uint16_t), 1024));
    cudaError_t e = gattn::launch_qkprep(qt, kb, positions, qtw, ktw, batch, seq_len, la, status, s);
    if (e != cudaSuccess) return fail_cuda(e, "query/key prologue launch");
    kt = ktw;
    qt = qtw;
  }
  gattn::PrefillArgs pa;
  pa.q = qt;
  pa.kt = kt;
  pa.v = la.k_eq_v ? kb : reinterpret_cast<const __nv_bfloat16*>(v_or_null);
  pa.out = reinterpret_cast<__nv_bfloat16*>(out);
  pa.B = batch;
  pa.S = seq_len;
  pa.status = status;
  pa.timeout_ns = gattn::wait_timeout_ns();
  pa.trace = static_cast<unsigned long long*>(g_trace_buf);
  pa.trace_bytes = g_trace_buf ? g_trace_bytes : 0;
  pa.seq_range = seq_range;
  if (g_prof_start) cudaEventRecord(g_prof_start, s);
  cudaError_t e = gattn::launch_prefill(pa, la, s);
  if (g_prof_stop) cudaEventRecord(g_prof_stop, s);
  if (e != cudaSuccess) return fail_cuda(e, "prefill launch");
  return GATTN_OK;
}

// ---- a chunk against a cached prefix ----------------------------------------------
size_t gattn_prefill_chunk_workspace_size(const gattn_cfg* cfg, int32_t batch, int32_t chunk_len, int32_t max_len) {
  gattn::LayerArgs la;
  if (resolve(cfg, &la, false) != GATTN_OK || batch < 0 || chunk_len < 0 || max_len < chunk_len) return 0;
  size_t bytes = kStatusBytes;
  if (prefill_needs_kprep(la))  // transformed cache keys, then the chunk's transformed queries
    bytes = round_up(bytes, 1024) +
            round_up(static_cast<size_t>(batch) * max_len * la.Hkv * la.D * sizeof(uint16_t), 1024) +
            static_cast<size_t>(batch) * chunk_len * la.H * la.D * sizeof(uint16_t);
  return bytes;
}

int gattn_kv_append(const gattn_bf16* k_new, const gattn_bf16* v_new_or_null, gattn_bf16* k_cache,
                    gattn_bf16* v_cache_or_null, const int32_t* cache_lens, int32_t batch, int32_t n_new,
                    int32_t max_len, int32_t num_kv_heads, int32_t head_dim, void* status_or_null,
                    gattn_stream stream) {
  g_last_error[0] = 0;
  if (batch < 0 || n_new < 0 || max_len < n_new || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 8)
    return fail(GATTN_ERR_INVALID_ARG, "need batch, n_new >= 0, max_len >= n_new, num_kv_heads > 0, head_dim % 8 == 0");
  if (batch == 0 || n_new == 0) return GATTN_OK;
  if (!k_new || !k_cache || !cache_lens) return fail(GATTN_ERR_INVALID_ARG, "k_new, k_cache and cache_lens must not be NULL");
  if ((v_new_or_null == nullptr) != (v_cache_or_null == nullptr))
    return fail(GATTN_ERR_INVALID_ARG, "v_new and v_cache must both be given or both be NULL");
  if (!aligned16(k_new) || !aligned16(k_cache) || (v_new_or_null && (!aligned16(v_new_or_null) ||
                                                                    !aligned16(v_cache_or_null))))
    return fail(GATTN_ERR_INVALID_ARG, "rows must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(cache_lens) & 3u) return fail(GATTN_ERR_INVALID_ARG, "cache_lens must be 4-byte aligned");
  if (status_or_null && !aligned16(status_or_null)) return fail(GATTN_ERR_INVALID_ARG, "status must be 16-byte aligned");
  cudaError_t e = gattn::launch_kv_append(
      reinterpret_cast<const __nv_bfloat16*>(k_new), reinterpret_cast<const __nv_bfloat16*>(v_new_or_null),
      reinterpret_cast<__nv_bfloat16*>(k_cache), reinterpret_cast<__nv_bfloat16*>(v_cache_or_null), cache_lens, batch,
      n_new, max_len, num_kv_heads, head_dim, static_cast<uint32_t*>(status_or_null),
      reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "kv append launch");
  return GATTN_OK;
}

int gattn_kv_append_layer(const gattn_cfg* cfg, const gattn_bf16* k_new, const gattn_bf16* v_new_or_null,
                          gattn_bf16* k_cache, gattn_bf16* v_cache_or_null, const int32_t* cache_lens,
                          int32_t batch, int32_t n_new, int32_t max_len, void* status_or_null,
                          gattn_stream stream) {
  g_last_error[0] = 0;
  gattn::LayerArgs la;
  int st = resolve(cfg, &la, true);
  if (st != GATTN_OK) return st;
  if (!la.kt_cache || !prefill_needs_kprep(la))
    return gattn_kv_append(k_new, v_new_or_null, k_cache, v_cache_or_null, cache_lens, batch, n_new, max_len, la.Hkv,
                           la.D, status_or_null, stream);
  if (batch < 0 || n_new < 0 || max_len < n_new)
    return fail(GATTN_ERR_INVALID_ARG, "need batch, n_new >= 0 and max_len >= n_new");
  if (batch == 0 || n_new == 0) return GATTN_OK;
  if (!k_new || !k_cache || !cache_lens || !v_new_or_null || !v_cache_or_null)
    return fail(GATTN_ERR_INVALID_ARG, "k_new, v_new, k_cache, v_cache and cache_lens must not be NULL");
  if (!aligned16(k_new) || !aligned16(k_cache) || !aligned16(v_new_or_null) || !aligned16(v_cache_or_null))
    return fail(GATTN_ERR_INVALID_ARG, "rows must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(cache_lens) & 3u) return fail(GATTN_ERR_INVALID_ARG, "cache_lens must be 4-byte aligned");
  if (status_or_null && !aligned16(status_or_null)) return fail(GATTN_ERR_INVALID_ARG, "status must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(status_or_null);
  cudaError_t e = gattn::launch_kv_append(nullptr, reinterpret_cast<const __nv_bfloat16*>(v_new_or_null),
                                          reinterpret_cast<__nv_bfloat16*>(k_cache),
                                          reinterpret_cast<__nv_bfloat16*>(v_cache_or_null), cache_lens, batch, n_new,
                                          max_len, la.Hkv, la.D, status, s);
  if (e == cudaSuccess)
    e = gattn::launch_key_append_transformed(reinterpret_cast<const __nv_bfloat16*>(k_new),
                                             reinterpret_cast<__nv_bfloat16*>(k_cache), cache_lens, batch, n_new,
                                             max_len, la, status, s);
  if (e != cudaSuccess) return fail_cuda(e, "kv append launch");
  return GATTN_OK;
}

int gattn_prefill_chunk(const gattn_bf16* q, const gattn_bf16* k_new_or_null, const gattn_bf16* v_new_or_null,
                        gattn_bf16* k_cache, gattn_bf16* v_cache_or_null, const int32_t* prefix_lens,
                        gattn_bf16* out, int32_t batch, int32_t chunk_len, int32_t max_len, const gattn_cfg* cfg,
                        void* workspace, size_t ws_bytes, gattn_stream stream) {
  g_last_error[0] = 0;
  gattn::LayerArgs la;
  int st = resolve(cfg, &la, true);
  if (st != GATTN_OK) return st;
  if (batch < 0 || chunk_len < 0 || max_len < chunk_len || max_len <= 0)
    return fail(GATTN_ERR_INVALID_ARG, "need batch, chunk_len >= 0 and max_len >= max(chunk_len, 1)");
  if (static_cast<long long>(batch) * max_len * la.H > (1LL << 31) - 1)
    return fail(GATTN_ERR_INVALID_ARG, "problem too large");
  if (!q || !k_cache || !out || !prefix_lens)
    return fail(GATTN_ERR_INVALID_ARG, "q, k_cache, prefix_lens and out must not be NULL");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(out))
    return fail(GATTN_ERR_INVALID_ARG, "q, k_cache and out must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(prefix_lens) & 3u)
    return fail(GATTN_ERR_INVALID_ARG, "prefix_lens must be 4-byte aligned");
  if (la.k_eq_v) {
    if ((v_cache_or_null && v_cache_or_null != k_cache) || (v_new_or_null && v_new_or_null != k_new_or_null))
      return fail(GATTN_ERR_INVALID_ARG, "k_eq_v: v_cache / v_new must be NULL or the key arrays");
  } else {
    if (!v_cache_or_null) return fail(GATTN_ERR_INVALID_ARG, "v_cache is NULL without k_eq_v");
    if (!aligned16(v_cache_or_null)) return fail(GATTN_ERR_INVALID_ARG, "v_cache must be 16-byte aligned");
    if ((k_new_or_null == nullptr) != (v_new_or_null == nullptr))
      return fail(GATTN_ERR_INVALID_ARG, "k_new and v_new must both be given or both be NULL");
  }
  if ((k_new_or_null && !aligned16(k_new_or_null)) || (v_new_or_null && !aligned16(v_new_or_null)))
    return fail(GATTN_ERR_INVALID_ARG, "k_new / v_new must be 16-byte aligned");
  const size_t need = gattn_prefill_chunk_workspace_size(cfg, batch, chunk_len, max_len);
  if (!workspace || ws_bytes < need) return fail(GATTN_ERR_WORKSPACE, "workspace missing or too small");
  if (!aligned16(workspace)) return fail(GATTN_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (batch == 0 || chunk_len == 0) return GATTN_OK;

  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  __nv_bfloat16* kc = reinterpret_cast<__nv_bfloat16*>(k_cache);
  __nv_bfloat16* vc = la.k_eq_v ? kc : reinterpret_cast<__nv_bfloat16*>(v_cache_or_null);
  // a transformed cache receives the chunk's keys normed and rotated, and its
  // keys are read as they are
  const bool kt_cache = la.kt_cache && prefill_needs_kprep(la);
  if (k_new_or_null) {
    cudaError_t e = gattn::launch_kv_append(
        kt_cache ? nullptr : reinterpret_cast<const __nv_bfloat16*>(k_new_or_null),
        la.k_eq_v ? nullptr : reinterpret_cast<const __nv_bfloat16*>(v_new_or_null), kc, la.k_eq_v ? nullptr : vc,
        prefix_lens, batch, chunk_len, max_len, la.Hkv, la.D, status, s);
    if (e == cudaSuccess && kt_cache)
      e = gattn::launch_key_append_transformed(reinterpret_cast<const __nv_bfloat16*>(k_new_or_null), kc, prefix_lens,
                                               batch, chunk_len, max_len, la, status, s);
    if (e != cudaSuccess) return fail_cuda(e, "kv append launch");
  }
  const __nv_bfloat16* kt = kc;
  const __nv_bfloat16* qt = reinterpret_cast<const __nv_bfloat16*>(q);
  if (prefill_needs_kprep(la)) {
    uint8_t* ws = static_cast<uint8_t*>(workspace);
    __nv_bfloat16* ktw = reinterpret_cast<__nv_bfloat16*>(ws + round_up(kStatusBytes, 1024));
    __nv_bfloat16* qtw = reinterpret_cast<__nv_bfloat16*>(
        ws + round_up(kStatusBytes, 1024) +
        round_up(static_cast<size_t>(batch) * max_len * la.Hkv * la.D * sizeof(uint16_t), 1024));
    cudaError_t e = gattn::launch_qkprep_chunk(qt, kc, prefix_lens, qtw, ktw, batch, chunk_len, max_len, la, status, s,
                                               !kt_cache);
    if (e != cudaSuccess) return fail_cuda(e, "query/key prologue launch");
    kt = kt_cache ? kc : ktw;
    qt = qtw;
  }
  gattn::PrefillArgs pa;
  pa.q = qt;
  pa.kt = kt;
  pa.v = vc;
  pa.out = reinterpret_cast<__nv_bfloat16*>(out);
  pa.B = batch;
  pa.S = chunk_len;
  pa.KV_S = max_len;
  pa.q_off = prefix_lens;
  pa.status = status;
  pa.timeout_ns = gattn::wait_timeout_ns();
  pa.trace = static_cast<unsigned long long*>(g_trace_buf);
  pa.trace_bytes = g_trace_buf ? g_trace_bytes : 0;
  if (g_prof_start) cudaEventRecord(g_prof_start, s);
  cudaError_t e = gattn::launch_prefill(pa, la, s);
  if (g_prof_stop) cudaEventRecord(g_prof_stop, s);
  if (e != cudaSuccess) return fail_cuda(e, "chunk prefill launch");
  return GATTN_OK;
}

// ---- decode ------------------------------------------------------------------------
static int decode_supported(const gattn::LayerArgs& la) {
  const int G = la.G;
  if (G != 1 && G != 2 && G != 4 && G != 8 && G != 16)
    return fail(GATTN_ERR_UNSUPPORTED, "decode supports num_heads / num_kv_heads in {1,2,4,8,16}");
  return GATTN_OK;
}

size_t gattn_decode_workspace_size(const gattn_cfg* cfg, int32_t batch, int32_t max_len) {
  gattn::LayerArgs la;
  if (resolve(cfg, &la, false) != GATTN_OK || batch < 0 || max_len <= 0) return 0;
  int nsplit, chunk;
  gattn::decode_plan(la, batch, max_len, &nsplit, &chunk);
  const size_t rows = static_cast<size_t>(batch) * la.H * nsplit;
  return round_up(kStatusBytes, 1024) + round_up(rows * la.D * sizeof(float), 1024) +
         rows * 2 * sizeof(float);
}

// The split plan, the workspace carve-up and the two launches of a decode call
// (da holds the cache pointers: bf16 k / v, or int8 kq / vq with their scales).
static int decode_launch(gattn::DecodeArgs& da, const gattn::LayerArgs& la, const gattn_bf16* q,
                         const int32_t* seq_lens, gattn_bf16* out, int32_t batch, int32_t max_len,
                         void* workspace, gattn_stream stream) {
  gattn::decode_plan(la, batch, max_len, &da.nsplit, &da.chunk);
  const size_t rows = static_cast<size_t>(batch) * la.H * da.nsplit;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  da.part_o = reinterpret_cast<float*>(ws + round_up(kStatusBytes, 1024));
  da.part_ml = reinterpret_cast<float*>(ws + round_up(kStatusBytes, 1024) +
                                        round_up(rows * la.D * sizeof(float), 1024));
  da.q = reinterpret_cast<const __nv_bfloat16*>(q);
  da.seq_lens = seq_lens;
  da.out = reinterpret_cast<__nv_bfloat16*>(out);
  da.B = batch;
  da.max_len = max_len;
  da.status = static_cast<uint32_t*>(workspace);
  da.trace = static_cast<unsigned long long*>(g_trace_buf);
  da.trace_bytes = g_trace_buf ? g_trace_bytes : 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (g_prof_start) cudaEventRecord(g_prof_start, s);
  cudaError_t e = gattn::launch_decode_split(da, la, s);
  if (g_prof_stop) cudaEventRecord(g_prof_stop, s);
  if (e != cudaSuccess) return fail_cuda(e, "decode split launch");
  e = gattn::launch_decode_combine(da, la, s);
  if (e != cudaSuccess) return fail_cuda(e, "decode combine launch");
  return GATTN_OK;
}

int gattn_decode(const gattn_bf16* q, const gattn_bf16* k_cache, const gattn_bf16* v_cache_or_null,
                 const int32_t* seq_lens, gattn_bf16* out, int32_t batch, int32_t max_len,
                 const gattn_cfg* cfg, void* workspace, size_t ws_bytes, gattn_stream stream) {
  g_last_error[0] = 0;
  gattn::LayerArgs la;
  int st = resolve(cfg, &la, true);
  if (st != GATTN_OK) return st;
  st = decode_supported(la);
  if (st != GATTN_OK) return st;
  if (batch < 0 || max_len <= 0) return fail(GATTN_ERR_INVALID_ARG, "batch must be >= 0 and max_len > 0");
  if (!q || !k_cache || !out || !seq_lens)
    return fail(GATTN_ERR_INVALID_ARG, "q, k_cache, seq_lens and out must not be NULL");
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(out))
    return fail(GATTN_ERR_INVALID_ARG, "q, k_cache and out must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(seq_lens) & 3u)
    return fail(GATTN_ERR_INVALID_ARG, "seq_lens must be 4-byte aligned");
  if (la.k_eq_v) {
    if (v_cache_or_null && v_cache_or_null != k_cache)
      return fail(GATTN_ERR_INVALID_ARG, "k_eq_v: v_cache must be NULL or k_cache");
  } else {
    if (!v_cache_or_null) return fail(GATTN_ERR_INVALID_ARG, "v_cache is NULL without k_eq_v");
    if (!aligned16(v_cache_or_null)) return fail(GATTN_ERR_INVALID_ARG, "v_cache must be 16-byte aligned");
  }
  const size_t need = gattn_decode_workspace_size(cfg, batch, max_len);
  if (!workspace || ws_bytes < need) return fail(GATTN_ERR_WORKSPACE, "workspace missing or too small");
  if (!aligned16(workspace)) return fail(GATTN_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (batch == 0) return GATTN_OK;

  gattn::DecodeArgs da;
  da.k = reinterpret_cast<const __nv_bfloat16*>(k_cache);
  da.v = la.k_eq_v ? da.k : reinterpret_cast<const __nv_bfloat16*>(v_cache_or_null);
  return decode_launch(da, la, q, seq_lens, out, batch, max_len, workspace, stream);
}

// ---- int8 KV cache -------------------------------------------------------------------
int gattn_kv_quantize(const gattn_bf16* x, int8_t* codes, float* scales, int64_t n_rows, int32_t head_dim,
                      gattn_stream stream) {
  g_last_error[0] = 0;
  if (head_dim != 256 && head_dim != 512) return fail(GATTN_ERR_UNSUPPORTED, "head_dim must be 256 or 512");
  if (n_rows < 0) return fail(GATTN_ERR_INVALID_ARG, "n_rows must be >= 0");
  if (n_rows == 0) return GATTN_OK;
  if (!x || !codes || !scales) return fail(GATTN_ERR_INVALID_ARG, "x, codes and scales must not be NULL");
  if (!aligned16(x) || !aligned16(codes)) return fail(GATTN_ERR_INVALID_ARG, "x and codes must be 16-byte aligned");
  if (reinterpret_cast<uintptr_t>(scales) & 3u) return fail(GATTN_ERR_INVALID_ARG, "scales must be 4-byte aligned");
  cudaError_t e = gattn::launch_kv_quantize(reinterpret_cast<const __nv_bfloat16*>(x), codes, scales, n_rows,
                                            head_dim, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail_cuda(e, "kv quantize launch");
  return GATTN_OK;
}

int gattn_decode_int8(const gattn_bf16* q, const int8_t* k_codes, const float* k_scales,
                      const int8_t* v_codes_or_null, const float* v_scales_or_null, const int32_t* seq_lens,
                      gattn_bf16* out, int32_t batch, int32_t max_len, const gattn_cfg* cfg, void* workspace,
                      size_t ws_bytes, gattn_stream stream) {
  g_last_error[0] = 0;
  gattn::LayerArgs la;
  int st = resolve(cfg, &la, true);
  if (st != GATTN_OK) return st;
  st = decode_supported(la);
  if (st != GATTN_OK) return st;
  if (batch < 0 || max_len <= 0) return fail(GATTN_ERR_INVALID_ARG, "batch must be >= 0 and max_len > 0");
  if (!q || !k_codes || !k_scales || !out || !seq_lens)
    return fail(GATTN_ERR_INVALID_ARG, "q, k_codes, k_scales, seq_lens and out must not be NULL");
  if (!aligned16(q) || !aligned16(k_codes) || !aligned16(out))
    return fail(GATTN_ERR_INVALID_ARG, "q, k_codes and out must be 16-byte aligned");
  if ((reinterpret_cast<uintptr_t>(seq_lens) & 3u) || (reinterpret_cast<uintptr_t>(k_scales) & 3u))
    return fail(GATTN_ERR_INVALID_ARG, "seq_lens and k_scales must be 4-byte aligned");
  if (la.k_eq_v) {
    if ((v_codes_or_null && v_codes_or_null != k_codes) || (v_scales_or_null && v_scales_or_null != k_scales))
      return fail(GATTN_ERR_INVALID_ARG, "k_eq_v: v_codes / v_scales must be NULL or the key arrays");
  } else {
    if (!v_codes_or_null || !v_scales_or_null)
      return fail(GATTN_ERR_INVALID_ARG, "v_codes / v_scales are NULL without k_eq_v");
    if (!aligned16(v_codes_or_null) || (reinterpret_cast<uintptr_t>(v_scales_or_null) & 3u))
      return fail(GATTN_ERR_INVALID_ARG, "v_codes must be 16-byte and v_scales 4-byte aligned");
  }
  const size_t need = gattn_decode_workspace_size(cfg, batch, max_len);
  if (!workspace || ws_bytes < need) return fail(GATTN_ERR_WORKSPACE, "workspace missing or too small");
  if (!aligned16(workspace)) return fail(GATTN_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  if (batch == 0) return GATTN_OK;
  gattn::DecodeArgs da;
  da.kq = k_codes;
  da.ks = k_scales;
  da.vq = la.k_eq_v ? k_codes : v_codes_or_null;
  da.vs = la.k_eq_v ? k_scales : v_scales_or_null;
  return decode_launch(da, la, q, seq_lens, out, batch, max_len, workspace, stream);
}

// ---- status ------------------------------------------------------------------------
int gattn_check(gattn_stream stream, void* workspace) {
  g_last_error[0] = 0;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail_cuda(e, "stream synchronize");
  if (!workspace) return fail(GATTN_ERR_INVALID_ARG, "workspace is NULL");
  uint32_t word = 0;
  e = cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail_cuda(e, "status read");
  if (word) {
    e = cudaMemsetAsync(workspace, 0, sizeof(word), s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return fail_cuda(e, "status clear");
  }
  if (word & 1u) return fail(GATTN_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  if (word & 2u) return fail(GATTN_ERR_DEVICE_BOUNDS, "a kernel saw an out-of-range position or length");
  return GATTN_OK;
}

void gattn_set_profile_events(void* start_event, void* stop_event) {
  if (start_event && stop_event) {
    g_prof_start = static_cast<cudaEvent_t>(start_event);
    g_prof_stop = static_cast<cudaEvent_t>(stop_event);
  } else {
    g_prof_start = nullptr;
    g_prof_stop = nullptr;
  }
}

void gattn_set_trace_buffer(void* device_buffer, size_t bytes) {
  g_trace_buf = (device_buffer && bytes) ? device_buffer : nullptr;
  g_trace_bytes = g_trace_buf ? bytes : 0;
}

int gattn_selftest_wait_timeout(void* workspace, size_t ws_bytes, uint32_t timeout_us,
                                gattn_stream stream) {
  g_last_error[0] = 0;
  if (!workspace || !aligned16(workspace)) return fail(GATTN_ERR_INVALID_ARG, "workspace NULL or misaligned");
  if (ws_bytes < kStatusBytes) return fail(GATTN_ERR_WORKSPACE, "workspace smaller than 256 bytes");
  if (timeout_us == 0 || timeout_us > 10000000u)
    return fail(GATTN_ERR_INVALID_ARG, "timeout_us must be in [1, 10^7]");
  cudaError_t e = gattn::launch_selftest_wait(static_cast<uint32_t*>(workspace),
                                              static_cast<uint64_t>(timeout_us) * 1000ull,
                                              reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? GATTN_OK : fail_cuda(e, "self-test launch");
}

}  // extern "C"
