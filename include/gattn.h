/*
 * libgattn -- Gemma 1-4 decoder self-attention forward on one NVIDIA B200 (sm_100a).
 *
 * The layer computed by both entry points, step by step:
 *   1. QK-norm: x / sqrt(mean(x^2) + eps) * g per head over head_dim, with
 *      g = 1 + w (Gemma 3's usual gain) or g = w (KerasFormers "Gemma 4",
 *      What changed: plain-weight RMSNorm).  QK-norm itself: Atlas "Gemma 4"
 *      summary (RMSNorm pre/post-norm + QK-norm).
 *   2. Rotary embedding on the first R = rotary_fraction * head_dim dims,
 *      rotate-half pairs (t, t + R/2), angle pos * theta^(-2t/F); dims past R
 *      pass through unchanged (KerasFormers "Gemma 4", What changed: zero-pad
 *      partial rope; KerasFormers "Gemma 3", What changed: dual RoPE bases).
 *   3. Logits s = (q~ . k~) * scalar^(-1/2) (ZeroModels "Gemma 2", API table:
 *      query_pre_attn_scalar).
 *   4. Optional cap s = c * tanh(s / c) (ZeroModels "Gemma 2", logit
 *      softcapping bullet).
 *   5. Causal mask, optionally a sliding window: key j is visible to query i
 *      iff j <= i and (window == 0 or i - j < window) on token indices
 *      (ZeroModels "Gemma 2", alternating attention bullet).
 *   6. Softmax over visible keys, weighted sum of values.  With k_eq_v the
 *      values are the raw key tensor (KerasFormers "Gemma 4", What changed:
 *      K=V global MQA with tied key and value projections).
 *   7. Query head h reads key/value head h / (num_heads / num_kv_heads)
 *      (GQA; MQA when num_kv_heads == 1: KerasFormers "Gemma", API table).
 *
 * Conventions for every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     allocates no device memory and keeps no state besides a per-device
 *     cache of attributes.  Pointers must be 16-byte aligned.
 *   - bf16 tensors are passed as gattn_bf16 (raw IEEE bfloat16 bits).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) and runs asynchronously; host arguments (cfg) are read during
 *     the call only.
 *   - Arguments are validated on the host before any launch; a failing check
 *     returns a gattn_status code and enqueues nothing.  Nothing aborts.
 *   - Errors found by the kernels themselves (a position outside the RoPE
 *     table, a sequence length outside [1, max_len], a bounded wait that ran
 *     out) are recorded in a status word at the start of the workspace and
 *     are read (and cleared) by gattn_check.
 */
#ifndef GATTN_H_
#define GATTN_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t gattn_bf16;        /* raw bfloat16 storage */
typedef struct CUstream_st* gattn_stream; /* same type as cudaStream_t */

typedef enum {
  GATTN_OK = 0,
  GATTN_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size or cfg field */
  GATTN_ERR_UNSUPPORTED = 2,   /* valid but not built (e.g. head_dim not 256/512) */
  GATTN_ERR_WORKSPACE = 3,     /* workspace missing or smaller than required */
  GATTN_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  GATTN_ERR_TIMEOUT = 5,       /* a kernel's bounded wait ran out (device) */
  GATTN_ERR_DEVICE_BOUNDS = 6  /* a kernel saw an out-of-range index (device) */
} gattn_status;

typedef enum {
  GATTN_NORM_NONE = 0,
  GATTN_NORM_ONE_PLUS_W = 1,   /* gain 1 + w */
  GATTN_NORM_W = 2             /* gain w */
} gattn_norm;

/* Layer description.  Read during the call only. */
typedef struct {
  int32_t num_heads;        /* H query heads                                    */
  int32_t num_kv_heads;     /* Hkv key/value heads; H % Hkv == 0                */
  int32_t head_dim;         /* D; 256 or 512                                    */
  int32_t window;           /* 0 = full causal; else keys with i - j < window   */
  float rope_theta;         /* RoPE base (1e4 local, 1e6 global)                */
  float rotary_fraction;    /* R = fraction * D rotated dims; 0 = no RoPE.
                               R must be a multiple of 16                       */
  int32_t rope_freq_dim;    /* F in theta^(-2t/F); 0 means head_dim             */
  const float* rope_table;  /* device table from gattn_rope_table_fill for the
                               same (theta, R, F); NULL iff R == 0              */
  int32_t rope_max_pos;     /* rows in rope_table; positions must be below it   */
  float softcap;            /* c > 0 caps logits at c * tanh(s / c); 0 = off    */
  float scalar;             /* query_pre_attn_scalar; scale = scalar^(-1/2) > 0 */
  int32_t k_eq_v;           /* 1: values are the key tensor (v pointer NULL or
                               equal to k)                                      */
  int32_t qk_norm;          /* gattn_norm                                       */
  float norm_eps;           /* RMSNorm epsilon (1e-6 in every Gemma card)       */
  const float* q_norm_w;    /* device fp32 [D], shared by heads; NULL iff NONE  */
  const float* k_norm_w;    /* device fp32 [D]; NULL iff NONE                   */
  int32_t keys_transformed; /* 0: KV caches hold raw keys.  1: caches hold the
                               keys after QK-norm and RoPE (each at its own
                               position), as gattn_kv_append_layer and
                               gattn_prefill_chunk's append write them; the
                               decode and chunk calls then skip the key
                               transforms.  Not with k_eq_v (values need the
                               raw keys).  gattn_prefill ignores it.            */
} gattn_cfg;

/* ---- RoPE table ---------------------------------------------------------
 * Table of (cos, sin) pairs, fp32, layout [max_pos][rot_dim/2][2], with
 * angle(p, t) = p * theta^(-2t/freq_dim) evaluated in double precision and
 * rounded once to fp32.  Build it once per (theta, rot_dim, freq_dim) and
 * pass it in gattn_cfg.rope_table.
 * gattn_rope_table_bytes returns 0 for invalid sizes.
 * gattn_rope_table_fill returns INVALID_ARG for a NULL/misaligned table,
 * theta <= 0, rot_dim odd or <= 0, freq_dim <= 0 or max_pos <= 0. */
size_t gattn_rope_table_bytes(int32_t max_pos, int32_t rot_dim);
int gattn_rope_table_fill(float* table, float theta, int32_t rot_dim, int32_t freq_dim,
                          int32_t max_pos, gattn_stream stream);

/* ---- workspace -----------------------------------------------------------
 * Every compute call takes a caller-owned device workspace.  Its first 256
 * bytes hold the status word; gattn_workspace_init zeroes them (call it once
 * after allocating).  Calls that share a workspace must be ordered on one
 * stream. */
int gattn_workspace_init(void* workspace, size_t ws_bytes, gattn_stream stream);

/* ---- prefill --------------------------------------------------------------
 * Self-attention of a whole prompt.
 *   q         [batch][seq_len][H][D]    bf16, row-major ("BSHD")
 *   k         [batch][seq_len][Hkv][D]  bf16
 *   v_or_null [batch][seq_len][Hkv][D]  bf16; NULL (or == k) when cfg->k_eq_v
 *   positions [batch][seq_len]          int32 RoPE positions, in [0, rope_max_pos)
 *                                       (may be NULL when R == 0)
 *   out       [batch][seq_len][H][D]    bf16, written completely
 * The mask works on token indices 0..seq_len-1; positions drive RoPE only.
 * workspace: at least gattn_prefill_workspace_size(cfg, batch, seq_len) bytes.
 * Returns GATTN_OK once the kernels are enqueued. */
size_t gattn_prefill_workspace_size(const gattn_cfg* cfg, int32_t batch, int32_t seq_len);
int gattn_prefill(const gattn_bf16* q, const gattn_bf16* k, const gattn_bf16* v_or_null,
                  const int32_t* positions, gattn_bf16* out, int32_t batch, int32_t seq_len,
                  const gattn_cfg* cfg, void* workspace, size_t ws_bytes, gattn_stream stream);

/* ---- prefill of a padded batch ------------------------------------------------
 * The same layer over a batch whose sequences are padded to seq_len: the
 * batched-prompt `attention_mask` (1 = keep, 0 = padding) of KerasFormers
 * "Gemma 4", Gemma4Generate.generate, given as each sequence's contiguous run
 * of valid tokens.
 *   seq_range [batch][2] int32 (device): valid tokens [lo, hi) of sequence b,
 *             0 <= lo <= hi <= seq_len (left padding: lo > 0; right: hi < seq_len).
 *             Values outside [0, seq_len] are clamped and flag
 *             GATTN_ERR_DEVICE_BOUNDS; lo >= hi makes the whole sequence padding.
 * A padding token is neither a query nor a key: key j is visible to query i
 * iff lo <= j <= i < hi (and i - j < window when windowed), and the output
 * rows of padding tokens are zero.  Positions of padding tokens must still be
 * in [0, rope_max_pos) (they are rotated, then ignored).  Every other argument,
 * the workspace size and the errors are those of gattn_prefill; with every
 * range [0, seq_len) the result is bit-identical to gattn_prefill's, except on
 * head_dim-512 layers with an even number of query heads per kv head, whose
 * whole prompts run on SM pairs (equal within rounding there).  Padding
 * rows of k and v get weight exactly 0 but are read: they must be finite. */
int gattn_prefill_padded(const gattn_bf16* q, const gattn_bf16* k, const gattn_bf16* v_or_null,
                         const int32_t* positions, const int32_t* seq_range, gattn_bf16* out,
                         int32_t batch, int32_t seq_len, const gattn_cfg* cfg, void* workspace,
                         size_t ws_bytes, gattn_stream stream);

/* ---- a chunk of a prompt against a cached prefix ------------------------------
 * The generate loop of KerasFormers "Gemma 4" (Gemma4Generate.generate) runs a
 * prompt, then tokens one by one, over a KV cache; a chunk is the step between:
 * C new tokens of sequence b at positions P_b .. P_b + C - 1 (P_b =
 * prefix_lens[b], the tokens already cached), each attending to the cache rows
 * [0, P_b + i] (within the window).  Caches hold RAW keys/values as in
 * gattn_decode, cached key j at position j.
 *   q               [batch][C][H][D] bf16, the chunk's queries (before QK-norm/RoPE)
 *   k_new, v_new    [batch][C][Hkv][D] bf16, the chunk's raw keys/values: copied into
 *                   cache rows [P_b, P_b + C) first (the cache append); both NULL
 *                   when those rows are already in the cache (v_new NULL with k_eq_v)
 *   k_cache, v_cache_or_null [batch][max_len][Hkv][D] bf16 (device, written by the append)
 *   prefix_lens     [batch] int32 (device): P_b in [0, max_len - C]; outside it is
 *                   clamped and flags GATTN_ERR_DEVICE_BOUNDS
 *   out             [batch][C][H][D] bf16
 * With C = the whole prompt and P_b = 0 it is gattn_prefill over the cache rows.
 * workspace: at least gattn_prefill_chunk_workspace_size(cfg, batch, C, max_len)
 * bytes (the transformed cache keys and chunk queries when QK-norm or RoPE is on).
 * Errors as gattn_prefill; the positions used by RoPE must be below rope_max_pos.
 * Cache rows past P_b + C are never weighted, but the last key tile of a chunk
 * reads up to 127 of them (weight exactly 0): they must hold finite values
 * (a zero-initialised cache does); rows beyond the tile are not read. */
size_t gattn_prefill_chunk_workspace_size(const gattn_cfg* cfg, int32_t batch, int32_t chunk_len, int32_t max_len);
int gattn_prefill_chunk(const gattn_bf16* q, const gattn_bf16* k_new_or_null, const gattn_bf16* v_new_or_null,
                        gattn_bf16* k_cache, gattn_bf16* v_cache_or_null, const int32_t* prefix_lens,
                        gattn_bf16* out, int32_t batch, int32_t chunk_len, int32_t max_len, const gattn_cfg* cfg,
                        void* workspace, size_t ws_bytes, gattn_stream stream);

/* gattn_kv_append: the cache append alone (e.g. before gattn_decode of a new token):
 * rows [batch][n_new][Hkv][D] bf16 of k_new (and v_new) into cache rows
 * [cache_lens[b], cache_lens[b] + n_new) of [batch][max_len][Hkv][D] caches.
 * cache_lens (device int32) are the rows held before the append; a value outside
 * [0, max_len - n_new] is clamped and, when status_or_null is a gattn workspace,
 * flags GATTN_ERR_DEVICE_BOUNDS there (read with gattn_check).  v_new and v_cache
 * are both NULL or both given; rows 16-byte aligned; head_dim a multiple of 8. */
int gattn_kv_append(const gattn_bf16* k_new, const gattn_bf16* v_new_or_null, gattn_bf16* k_cache,
                    gattn_bf16* v_cache_or_null, const int32_t* cache_lens, int32_t batch, int32_t n_new,
                    int32_t max_len, int32_t num_kv_heads, int32_t head_dim, void* status_or_null,
                    gattn_stream stream);

/* gattn_kv_append_layer: the append of gattn_kv_append for a layer: with
 * cfg->keys_transformed the key rows are written after QK-norm and RoPE at their
 * positions cache_lens[b] + s (the rows a transformed cache holds), the values
 * raw; otherwise it is gattn_kv_append.  cache_lens out of range are clamped and
 * flag GATTN_ERR_DEVICE_BOUNDS in status_or_null (a gattn workspace), as are
 * positions past the RoPE table. */
int gattn_kv_append_layer(const gattn_cfg* cfg, const gattn_bf16* k_new, const gattn_bf16* v_new_or_null,
                          gattn_bf16* k_cache, gattn_bf16* v_cache_or_null, const int32_t* cache_lens,
                          int32_t batch, int32_t n_new, int32_t max_len, void* status_or_null,
                          gattn_stream stream);

/* ---- context parallelism: one long prompt over several GPUs --------------------
 * The model cards give Gemma 4 a 256K context window (KerasFormers "Gemma 4"),
 * and the Atlas "Gemma 4" summary trains with the data sharded by sequence as
 * well as by batch and replica; one prompt that long is split over the GPUs of
 * a node by query rows.  gattn_cp_blocks is the split: the prompt's seq_len
 * tokens are cut into 2 * world contiguous blocks as evenly as possible (the
 * first seq_len mod (2 * world) blocks one token longer), and rank r owns
 * blocks r and 2 * world - 1 - r, so that every rank's causal work (the
 * visible pairs of its query rows) is the same to within one block's rows.
 * Each rank then gathers every rank's key (and value) rows of its blocks (one
 * all-gather over the node's links; with k_eq_v one tensor), and runs each of
 * its two blocks as a chunk (gattn_prefill_chunk with the gathered keys as the
 * cache, prefix_lens = the block's first token, no append): a block's rows
 * see exactly the keys a whole-prompt prefill gives them.
 * Writes starts[0..1] and lens[0..1] (host int32): rank's two blocks in token
 * order.  Host only; returns GATTN_OK, or GATTN_ERR_INVALID_ARG for world < 1,
 * rank outside [0, world), seq_len < 0 or NULL pointers. */
int gattn_cp_blocks(int32_t seq_len, int32_t world, int32_t rank, int32_t* starts, int32_t* lens);

/* ---- decode ----------------------------------------------------------------
 * One decode step: query b (at position seq_lens[b]-1) against cache rows
 * [0, seq_lens[b]) of its own cache.  Caches hold RAW keys/values (before
 * QK-norm and RoPE), or transformed keys with cfg->keys_transformed; cached key
 * j sits at position j.
 *   q               [batch][H][D]            bf16
 *   k_cache         [batch][max_len][Hkv][D] bf16
 *   v_cache_or_null [batch][max_len][Hkv][D] bf16; NULL (or == k_cache) when k_eq_v
 *   seq_lens        [batch] int32 in [1, max_len] (device); rows outside it write zeros
 *                   and flag GATTN_ERR_DEVICE_BOUNDS
 *   out             [batch][H][D]            bf16
 * Only the visible rows (the last `window` rows when windowed) are read.
 * workspace: at least gattn_decode_workspace_size(cfg, batch, max_len) bytes. */
size_t gattn_decode_workspace_size(const gattn_cfg* cfg, int32_t batch, int32_t max_len);
int gattn_decode(const gattn_bf16* q, const gattn_bf16* k_cache, const gattn_bf16* v_cache_or_null,
                 const int32_t* seq_lens, gattn_bf16* out, int32_t batch, int32_t max_len,
                 const gattn_cfg* cfg, void* workspace, size_t ws_bytes, gattn_stream stream);

/* ---- int8 KV cache ------------------------------------------------------------
 * The Atlas summary of the Gemma 4 report offers int8 KV caching (Table 3, "+KV"
 * at 32k context) without giving the format.  Here: every cache row (the
 * head_dim values of one position and one kv head) is stored as int8 codes c and
 * one fp32 scale s, dequantised as c * s; s = max|x| / 127 and
 * c = round-half-even(x / s) clipped to [-127, 127], both divisions in IEEE
 * float32 (a row of zeros: s = 0, codes 0).  Inputs must be finite.
 *
 * gattn_kv_quantize: x [n_rows][head_dim] bf16 -> codes [n_rows][head_dim]
 * int8 and scales [n_rows] fp32 (all device; a [batch][len][Hkv][D] cache is
 * n_rows = batch * len * Hkv).  head_dim 256 or 512 (else
 * GATTN_ERR_UNSUPPORTED); x and codes 16-byte aligned, scales 4-byte aligned.
 * The codes and scales equal a float32 evaluation of the definition bit for bit.
 * Enqueued on `stream`; no workspace, no status word. */
int gattn_kv_quantize(const gattn_bf16* x, int8_t* codes, float* scales, int64_t n_rows, int32_t head_dim,
                      gattn_stream stream);

/* gattn_decode_int8: gattn_decode over an int8 cache, computing with the
 * dequantised rows (the same RAW keys/values as gattn_decode's caches).
 *   k_codes / v_codes   [batch][max_len][Hkv][D] int8, 16-byte aligned
 *   k_scales / v_scales [batch][max_len][Hkv] fp32, 4-byte aligned
 *   with k_eq_v: v_codes / v_scales NULL (or the key arrays); values are the
 *   dequantised raw keys.
 * Every other argument, the workspace size (gattn_decode_workspace_size) and
 * the errors are those of gattn_decode, and so are the layers it takes: 1, 2 or
 * 4 query heads per kv head (head_dim 512: 1 or 2, and 1, 2, 4 or 8 kv heads)
 * run the persistent CUDA-core split kernel; K=V layers with 8 or 16 query
 * heads per kv head (the Gemma 4 global layer) the tensor-core kernel, whose
 * MMAs take the codes themselves (integers, exact in fp16) and apply each row's
 * scale to its logits and its softmax weights; the rest a slower CUDA-core split
 * kernel that dequantises row by row. */
int gattn_decode_int8(const gattn_bf16* q, const int8_t* k_codes, const float* k_scales,
                      const int8_t* v_codes_or_null, const float* v_scales_or_null, const int32_t* seq_lens,
                      gattn_bf16* out, int32_t batch, int32_t max_len, const gattn_cfg* cfg, void* workspace,
                      size_t ws_bytes, gattn_stream stream);

/* ---- decode without a workspace ----------------------------------------------------
 * The model cards describe no such call; it exists for callers that cannot
 * allocate device memory at the point where they decode: code running inside
 * an allocator-free or pre-planned memory region (e.g. a serving loop whose
 * pool is fixed up front), or code that must not call cudaMalloc while other
 * work is in flight.  It computes exactly what gattn_decode computes, with the
 * same arguments minus the workspace, and calls no cudaMalloc, cudaFree or any
 * allocating routine.
 * Its split partials live in a 16 MiB device array inside the library, which
 * every GPU that loads the library holds until the process exits.  The first
 * call on each device looks up that array's device address
 * (cudaGetSymbolAddress) with the device current; make that first call before
 * any stream capture.  Calls share the array: two calls whose work overlaps on
 * the GPU (different streams, or different host threads on one device) race
 * and may return wrong results; order them on one stream.  Nothing in the
 * array needs to start at zero (every partial is written before it is read),
 * and it keeps the last call's partials.
 * A split slot takes batch * num_heads * (head_dim + 2) * 4 bytes.  When the
 * normal split count would not fit, it uses fewer, longer splits; if even the
 * layer's smallest plan does not fit (one slot per chunk, and, on layers with
 * 1, 2 or 4 query heads per kv head, which run on the CUDA-core kernel,
 * 8 / num_kv_heads slots per chunk), it returns GATTN_ERR_UNSUPPORTED and
 * enqueues nothing.  There is no status word, so nothing device-side is
 * reported: kernel-side range errors (a seq_lens entry outside [1, max_len],
 * a position past the RoPE table) are handled as gattn_decode handles them
 * (rows written as zeros / positions clamped), and if a kernel's bounded wait
 * runs out (the 2 s default of gattn_set_wait_timeout_us), the key chunk that
 * split was reading is left out of the merge: the call returns a finite but
 * wrong result for that row without any error. */
int gattn_decode_noalloc(const gattn_bf16* q, const gattn_bf16* k_cache,
                         const gattn_bf16* v_cache_or_null, const int32_t* seq_lens, gattn_bf16* out,
                         int32_t batch, int32_t max_len, const gattn_cfg* cfg, gattn_stream stream);

/* ---- status --------------------------------------------------------------------
 * gattn_check synchronises `stream`, reads and clears the workspace status
 * word, and returns GATTN_ERR_TIMEOUT or GATTN_ERR_DEVICE_BOUNDS if a kernel
 * recorded one since the last check (timeout wins), else GATTN_OK (or
 * GATTN_ERR_CUDA if synchronising failed). */
int gattn_check(gattn_stream stream, void* workspace);
const char* gattn_status_string(int status);
/* Message for the last failing call on this host thread ("" if none). */
const char* gattn_last_error(void);

/* ---- self-test hooks ----------------------------------------------------------
 * gattn_selftest_wait_timeout launches one CTA that waits, with the library's
 * bounded-wait helper and a limit of `timeout_us` microseconds, on an
 * mbarrier that nothing ever arrives on; the wait runs out, the CTA records
 * GATTN_ERR_TIMEOUT in the workspace status word and exits normally.  It lets
 * a test check the timeout path without hanging or faulting a GPU.
 * gattn_set_wait_timeout_us sets the limit every later kernel launch in this
 * process uses for its mbarrier waits (default 2,000,000 us); 0 restores it. */
int gattn_selftest_wait_timeout(void* workspace, size_t ws_bytes, uint32_t timeout_us,
                                gattn_stream stream);
void gattn_set_wait_timeout_us(uint32_t timeout_us);

/* ---- profiling hook ----------------------------------------------------------
 * gattn_set_profile_events(start, stop): when both are non-NULL (cudaEvent_t
 * handles), every later gattn_prefill / gattn_decode call on this host thread
 * records `start` on its stream right before launching its main kernel (the
 * tensor-core prefill kernel, or the decode split kernel) and `stop` right
 * after it, so a caller can time that kernel alone with cudaEventElapsedTime.
 * Passing NULLs turns it off.  The events stay owned by the caller. */
void gattn_set_profile_events(void* start_event, void* stop_event);

/* gattn_set_trace_buffer(buf, bytes): when buf (a device buffer of `bytes`
 * bytes, 8-byte aligned) is non-NULL, every later gattn_prefill call on this
 * host thread has each of its first bytes/4096 CTAs write a timeline of 512
 * 64-bit entries: [0] start time (ns, %globaltimer), [1] SM id, [2] key tiles,
 * [3] Q ready, [4] epilogue start, [5] end, [6] first key box landed, and per
 * key tile j < 120: [8+j] S(j) seen by the softmax, [128+j] P(j) written,
 * [248+j] Q K^T(j) issued, [368+j] P V(j) issued, each in ns after [0].
 * Whole prompts of head_dim-512 layers with an even number of query heads per
 * kv head run on SM pairs: there CTA i of the first bytes/4096 writes [0]
 * start, [1] SM id, [2] its rank in the pair, [3] items it takes, [4] key
 * tiles of its first item, and per key tile j < 120 of that item [8+j] S(j)
 * seen by the softmax, [128+j] P(j) written, and (first CTA of the pair)
 * [248+j] Q K^T(j) issued, [368+j] P V(j) issued.
 * A debugging aid; NULL turns it off. */
void gattn_set_trace_buffer(void* device_buffer, size_t bytes);

/* Library version string, e.g. "libgattn 0.1 sm_100a". */
const char* gattn_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GATTN_H_ */
