"""libgattn: Gemma 1-4 decoder self-attention forward on one B200 (sm_100a).

The compute lives in ``libgattn.so`` (C ABI in ``include/gattn.h``); this
package holds its ctypes binding (``gattn``) and build script (``build``).
"""
from .gattn import (AttentionLayer, GattnCfg, GattnError, LayerSpec, check, kv_append, kv_quantize, lib, rope_table,
                    selftest_wait_timeout, set_profile_events, set_wait_timeout_us, version)

__all__ = ["AttentionLayer", "GattnCfg", "GattnError", "LayerSpec", "check", "kv_append", "kv_quantize", "lib", "rope_table",
           "selftest_wait_timeout", "set_profile_events", "set_wait_timeout_us", "version"]
