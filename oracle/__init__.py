"""Float64 CPU oracle (test infrastructure only; see ``oracle.oracle``)."""
from .oracle import (NORM_NONE, NORM_ONE_PLUS_W, NORM_W, attention_decode,
                     attention_decode_int8, attention_prefill, attention_prefill_chunk, chunk_partial, kv_dequantize,
                     kv_quantize, lse_merge, rms_norm, rope, rope_angles, softcap, transform_keys, visible)

__all__ = ["NORM_NONE", "NORM_ONE_PLUS_W", "NORM_W", "attention_decode",
           "attention_decode_int8", "attention_prefill", "attention_prefill_chunk", "chunk_partial", "kv_dequantize",
           "kv_quantize", "lse_merge", "rms_norm", "rope", "rope_angles", "softcap", "transform_keys", "visible"]
