"""The C ABI: the library loads, exports every function the header declares,
and rejects bad arguments on the host before any launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

import gemma_family_decoder_b200 as G
from gemma_family_decoder_b200 import gattn

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gattn.h")
ALIGNED = 0x10000  # a fake, 16-byte aligned device address: never dereferenced here


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gattn_[a-z_0-9]+)\s*\(", text)))


def test_header_and_exports_agree():
    L = G.lib()
    names = declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(gattn.EXPORTS)


def test_cfg_struct_matches_header_layout():
    # int32 x4, float x2, int32, (pad), ptr, int32, float x2, int32 x2, float, ptr x2, int32, (pad)
    assert ctypes.sizeof(G.GattnCfg) == 88
    assert G.GattnCfg.keys_transformed.offset == 80
    assert G.GattnCfg.rope_table.offset == 32
    assert G.GattnCfg.q_norm_w.offset == 64


def cfg(**kw):
    base = dict(num_heads=8, num_kv_heads=1, head_dim=256, window=0, rope_theta=1e4,
                rotary_fraction=0.0, rope_freq_dim=0, rope_table=None, rope_max_pos=0,
                softcap=0.0, scalar=256.0, k_eq_v=0, qk_norm=0, norm_eps=1e-6,
                q_norm_w=None, k_norm_w=None)
    base.update(kw)
    return G.GattnCfg(**base)


def prefill(c, q=ALIGNED, k=ALIGNED, v=ALIGNED, pos=ALIGNED, out=ALIGNED, B=1, S=16, ws=ALIGNED,
            ws_bytes=1 << 30):
    return G.lib().gattn_prefill(q, k, v, pos, out, B, S, ctypes.byref(c), ws, ws_bytes, None)


def decode(c, q=ALIGNED, k=ALIGNED, v=ALIGNED, lens=ALIGNED, out=ALIGNED, B=1, Lmax=16, ws=ALIGNED,
           ws_bytes=1 << 30):
    return G.lib().gattn_decode(q, k, v, lens, out, B, Lmax, ctypes.byref(c), ws, ws_bytes, None)


INVALID, UNSUPPORTED, WORKSPACE = 1, 2, 3


@pytest.mark.parametrize("over,code", [
    (dict(head_dim=128), UNSUPPORTED),
    (dict(num_heads=6, num_kv_heads=4), INVALID),
    (dict(num_kv_heads=0), INVALID),
    (dict(window=-1), INVALID),
    (dict(rotary_fraction=0.25), INVALID),          # RoPE on without a table
    (dict(rotary_fraction=0.3), INVALID),           # 76.8 dims
    (dict(rotary_fraction=0.375), UNSUPPORTED),     # 96 dims: not a power of two
    (dict(softcap=-1.0), INVALID),
    (dict(scalar=0.0), INVALID),
    (dict(qk_norm=3), INVALID),
    (dict(qk_norm=1), INVALID),                     # weights missing
    (dict(k_eq_v=2), INVALID),
    (dict(keys_transformed=2), INVALID),
    (dict(keys_transformed=1, k_eq_v=1), INVALID),     # tied values need the raw keys
])
def test_prefill_rejects_bad_cfg(over, code):
    assert prefill(cfg(**over)) == code
    assert G.lib().gattn_last_error()


def test_prefill_rejects_bad_pointers_and_sizes():
    c = cfg()
    assert prefill(c, q=None) == INVALID
    assert prefill(c, q=ALIGNED + 8) == INVALID
    assert prefill(c, v=None) == INVALID
    assert prefill(c, B=-1) == INVALID
    assert prefill(c, ws=None) == WORKSPACE
    assert prefill(c, ws_bytes=16) == WORKSPACE
    ck = cfg(k_eq_v=1)
    assert prefill(ck, v=ALIGNED + 4096) == INVALID  # tied keys/values but a different v
    cr = cfg(rotary_fraction=1.0, rope_table=ALIGNED, rope_max_pos=64)
    assert prefill(cr, pos=None) == INVALID


def prefill_padded(c, sr=ALIGNED, B=1, S=16, **kw):
    a = dict(q=ALIGNED, k=ALIGNED, v=ALIGNED, pos=ALIGNED, out=ALIGNED, ws=ALIGNED, ws_bytes=1 << 30)
    a.update(kw)
    return G.lib().gattn_prefill_padded(a["q"], a["k"], a["v"], a["pos"], sr, a["out"], B, S, ctypes.byref(c),
                                        a["ws"], a["ws_bytes"], None)


def test_prefill_padded_rejects_bad_args():
    c = cfg()
    assert prefill_padded(c, sr=None) == INVALID
    assert prefill_padded(c, sr=ALIGNED + 2) == INVALID      # int32 pairs: 4-byte aligned
    assert prefill_padded(c, q=ALIGNED + 8) == INVALID       # then every check of gattn_prefill
    assert prefill_padded(c, ws_bytes=16) == WORKSPACE
    assert prefill_padded(cfg(head_dim=128)) == UNSUPPORTED
    assert prefill_padded(c, B=0) == 0
    assert G.lib().gattn_last_error() == b""


def test_kv_quantize_rejects_bad_args():
    L = G.lib()
    assert L.gattn_kv_quantize(ALIGNED, ALIGNED, ALIGNED, 4, 128, None) == UNSUPPORTED
    assert L.gattn_kv_quantize(ALIGNED, ALIGNED, ALIGNED, -1, 256, None) == INVALID
    assert L.gattn_kv_quantize(None, ALIGNED, ALIGNED, 4, 256, None) == INVALID
    assert L.gattn_kv_quantize(ALIGNED + 8, ALIGNED, ALIGNED, 4, 256, None) == INVALID
    assert L.gattn_kv_quantize(ALIGNED, ALIGNED, ALIGNED + 2, 4, 256, None) == INVALID
    assert L.gattn_kv_quantize(ALIGNED, ALIGNED, ALIGNED, 0, 256, None) == 0   # nothing to do


def decode_int8(c, q=ALIGNED, kc=ALIGNED, ks=ALIGNED, vc=ALIGNED, vs=ALIGNED, lens=ALIGNED, out=ALIGNED, B=1,
                Lmax=16, ws=ALIGNED, ws_bytes=1 << 30):
    return G.lib().gattn_decode_int8(q, kc, ks, vc, vs, lens, out, B, Lmax, ctypes.byref(c), ws, ws_bytes, None)


def test_decode_int8_rejects_bad_args():
    c = cfg(num_heads=16, num_kv_heads=8)
    assert decode_int8(cfg(num_heads=24, num_kv_heads=1)) == UNSUPPORTED   # group of 24, as gattn_decode
    assert decode_int8(c, kc=None) == INVALID
    assert decode_int8(c, ks=ALIGNED + 2) == INVALID
    assert decode_int8(c, kc=ALIGNED + 4) == INVALID
    assert decode_int8(c, vs=None) == INVALID                              # separate values need scales
    ck = cfg(num_heads=4, num_kv_heads=2, k_eq_v=1)
    assert decode_int8(ck, vc=ALIGNED + 4096, vs=None) == INVALID         # tied: v arrays NULL or the key ones
    assert decode_int8(ck, vc=None, vs=None, B=0) == 0
    assert decode_int8(c, ws_bytes=16) == WORKSPACE
    assert decode_int8(c, B=0) == 0


def prefill_chunk(c, q=ALIGNED, kn=ALIGNED, vn=ALIGNED, kc=ALIGNED, vc=ALIGNED, pre=ALIGNED, out=ALIGNED, B=1, C=16,
                  Lmax=64, ws=ALIGNED, ws_bytes=1 << 30):
    return G.lib().gattn_prefill_chunk(q, kn, vn, kc, vc, pre, out, B, C, Lmax, ctypes.byref(c), ws, ws_bytes, None)


def test_prefill_chunk_rejects_bad_args():
    c = cfg()
    assert prefill_chunk(c, C=65) == INVALID                    # chunk longer than the cache
    assert prefill_chunk(c, pre=None) == INVALID
    assert prefill_chunk(c, pre=ALIGNED + 2) == INVALID
    assert prefill_chunk(c, kc=ALIGNED + 8) == INVALID
    assert prefill_chunk(c, vn=None) == INVALID                  # k_new without v_new
    assert prefill_chunk(c, vc=None) == INVALID
    assert prefill_chunk(cfg(head_dim=128)) == UNSUPPORTED
    assert prefill_chunk(c, ws_bytes=16) == WORKSPACE
    assert prefill_chunk(c, B=0) == 0 and prefill_chunk(c, C=0) == 0
    assert prefill_chunk(c, kn=None, vn=None, B=0) == 0
    ck = cfg(k_eq_v=1)
    assert prefill_chunk(ck, vc=ALIGNED + 4096) == INVALID      # tied: v_cache NULL or k_cache
    n_small = G.lib().gattn_prefill_chunk_workspace_size(ctypes.byref(c), 2, 16, 64)
    cr = cfg(rotary_fraction=1.0, rope_table=ALIGNED, rope_max_pos=64)
    n_rope = G.lib().gattn_prefill_chunk_workspace_size(ctypes.byref(cr), 2, 16, 64)
    assert n_small >= 4 and n_rope >= 2 * 64 * 1 * 256 * 2 + 2 * 16 * 8 * 256 * 2
    assert G.lib().gattn_prefill_chunk_workspace_size(ctypes.byref(c), 2, 65, 64) == 0


def test_kv_append_rejects_bad_args():
    L = G.lib()
    f = L.gattn_kv_append
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 1, 17, 16, 2, 256, None, None) == INVALID  # n_new > max_len
    assert f(ALIGNED, None, ALIGNED, ALIGNED, ALIGNED, 1, 4, 16, 2, 256, None, None) == INVALID   # v_new xor v_cache
    assert f(ALIGNED + 8, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 1, 4, 16, 2, 256, None, None) == INVALID
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED + 2, 1, 4, 16, 2, 256, None, None) == INVALID
    assert f(ALIGNED, ALIGNED, ALIGNED, ALIGNED, ALIGNED, 1, 4, 16, 2, 100, None, None) == INVALID  # head_dim % 8
    assert f(None, None, None, None, None, 0, 4, 16, 2, 256, None, None) == 0                    # empty


def test_empty_problem_is_a_no_op():
    assert prefill(cfg(), B=0) == 0
    assert prefill(cfg(), S=0) == 0
    assert decode(cfg(), B=0) == 0


def test_decode_rejects_bad_args():
    assert decode(cfg(num_heads=24, num_kv_heads=1)) == UNSUPPORTED   # group of 24
    assert decode(cfg(), lens=None) == INVALID
    assert decode(cfg(), Lmax=0) == INVALID
    assert decode(cfg(), ws_bytes=8) == WORKSPACE


def test_workspace_sizes():
    L = G.lib()
    c = cfg(rotary_fraction=1.0, rope_table=ALIGNED, rope_max_pos=2048)
    n = L.gattn_prefill_workspace_size(ctypes.byref(c), 4, 2048)
    assert n >= 4 * 2048 * 1 * 256 * 2            # transformed keys
    assert L.gattn_prefill_workspace_size(ctypes.byref(cfg()), 4, 2048) >= 256
    assert L.gattn_prefill_workspace_size(ctypes.byref(cfg(head_dim=100)), 4, 2048) == 0
    assert L.gattn_decode_workspace_size(ctypes.byref(cfg()), 64, 32768) > 0
    assert L.gattn_rope_table_bytes(32768, 128) == 32768 * 64 * 8
    assert L.gattn_rope_table_bytes(16, 3) == 0


def test_status_strings():
    L = G.lib()
    for code in range(7):
        assert L.gattn_status_string(code)
    assert G.version().startswith("libgattn")


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    # no fallback of any kind: without libgattn.so every call raises
    monkeypatch.setattr(gattn, "_lib", None)
    monkeypatch.setattr(gattn, "LIB_PATH", str(tmp_path / "absent" / "libgattn.so"))
    with pytest.raises(ImportError):
        gattn.lib()
