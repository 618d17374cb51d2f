"""Thin ctypes binding of libgattn (argument marshalling only).

Every function here forwards torch tensors' device pointers and the current
CUDA stream to the C ABI declared in ``include/gattn.h``; all arithmetic runs
in the library's CUDA kernels.  There is no fallback: if ``libgattn.so`` is
missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgattn.so")

GATTN_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "WORKSPACE", 4: "CUDA",
                5: "TIMEOUT", 6: "DEVICE_BOUNDS"}

NORM_NONE, NORM_ONE_PLUS_W, NORM_W = 0, 1, 2

EXPORTS = ("gattn_version", "gattn_status_string", "gattn_last_error", "gattn_rope_table_bytes",
           "gattn_rope_table_fill", "gattn_workspace_init", "gattn_prefill_workspace_size",
           "gattn_prefill", "gattn_decode_workspace_size", "gattn_decode", "gattn_check",
           "gattn_selftest_wait_timeout", "gattn_set_wait_timeout_us", "gattn_set_profile_events",
           "gattn_set_trace_buffer", "gattn_decode_noalloc", "gattn_prefill_padded", "gattn_kv_quantize",
           "gattn_decode_int8", "gattn_prefill_chunk_workspace_size", "gattn_prefill_chunk", "gattn_kv_append",
           "gattn_kv_append_layer", "gattn_cp_blocks")


class GattnError(RuntimeError):
    def __init__(self, status: int, where: str, msg: str):
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)} ({msg})")
        self.status = status


class GattnCfg(ctypes.Structure):
    """Mirror of ``gattn_cfg`` (include/gattn.h)."""
    _fields_ = [
        ("num_heads", ctypes.c_int32),
        ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("window", ctypes.c_int32),
        ("rope_theta", ctypes.c_float),
        ("rotary_fraction", ctypes.c_float),
        ("rope_freq_dim", ctypes.c_int32),
        ("rope_table", ctypes.c_void_p),
        ("rope_max_pos", ctypes.c_int32),
        ("softcap", ctypes.c_float),
        ("scalar", ctypes.c_float),
        ("k_eq_v", ctypes.c_int32),
        ("qk_norm", ctypes.c_int32),
        ("norm_eps", ctypes.c_float),
        ("q_norm_w", ctypes.c_void_p),
        ("k_norm_w", ctypes.c_void_p),
        ("keys_transformed", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgattn.so (built by ``python -m gemma_family_decoder_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libgattn.so not found at {LIB_PATH}; build it with "
                              "`python -m gemma_family_decoder_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, i32, f32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32, ctypes.c_float
        L.gattn_version.restype = ctypes.c_char_p
        L.gattn_status_string.restype = ctypes.c_char_p
        L.gattn_status_string.argtypes = [ctypes.c_int]
        L.gattn_last_error.restype = ctypes.c_char_p
        L.gattn_rope_table_bytes.restype = sz
        L.gattn_rope_table_bytes.argtypes = [i32, i32]
        L.gattn_rope_table_fill.restype = ctypes.c_int
        L.gattn_rope_table_fill.argtypes = [vp, f32, i32, i32, i32, vp]
        L.gattn_workspace_init.restype = ctypes.c_int
        L.gattn_workspace_init.argtypes = [vp, sz, vp]
        L.gattn_prefill_workspace_size.restype = sz
        L.gattn_prefill_workspace_size.argtypes = [ctypes.POINTER(GattnCfg), i32, i32]
        L.gattn_prefill.restype = ctypes.c_int
        L.gattn_prefill.argtypes = [vp, vp, vp, vp, vp, i32, i32, ctypes.POINTER(GattnCfg), vp, sz, vp]
        L.gattn_decode_workspace_size.restype = sz
        L.gattn_decode_workspace_size.argtypes = [ctypes.POINTER(GattnCfg), i32, i32]
        L.gattn_decode.restype = ctypes.c_int
        L.gattn_decode.argtypes = [vp, vp, vp, vp, vp, i32, i32, ctypes.POINTER(GattnCfg), vp, sz, vp]
        L.gattn_check.restype = ctypes.c_int
        L.gattn_check.argtypes = [vp, vp]
        L.gattn_selftest_wait_timeout.restype = ctypes.c_int
        L.gattn_selftest_wait_timeout.argtypes = [vp, sz, ctypes.c_uint32, vp]
        L.gattn_set_wait_timeout_us.restype = None
        L.gattn_set_wait_timeout_us.argtypes = [ctypes.c_uint32]
        L.gattn_set_profile_events.restype = None
        L.gattn_set_profile_events.argtypes = [vp, vp]
        L.gattn_set_trace_buffer.restype = None
        L.gattn_set_trace_buffer.argtypes = [vp, sz]
        L.gattn_decode_noalloc.restype = ctypes.c_int
        L.gattn_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i32, i32, ctypes.POINTER(GattnCfg), vp]
        L.gattn_prefill_chunk_workspace_size.restype = sz
        L.gattn_prefill_chunk_workspace_size.argtypes = [ctypes.POINTER(GattnCfg), i32, i32, i32]
        L.gattn_prefill_chunk.restype = ctypes.c_int
        L.gattn_prefill_chunk.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, ctypes.POINTER(GattnCfg), vp, sz,
                                          vp]
        L.gattn_kv_append_layer.restype = ctypes.c_int
        L.gattn_kv_append_layer.argtypes = [ctypes.POINTER(GattnCfg), vp, vp, vp, vp, vp, i32, i32, i32, vp, vp]
        L.gattn_kv_append.restype = ctypes.c_int
        L.gattn_kv_append.argtypes = [vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]
        L.gattn_kv_quantize.restype = ctypes.c_int
        L.gattn_kv_quantize.argtypes = [vp, vp, vp, ctypes.c_int64, i32, vp]
        L.gattn_decode_int8.restype = ctypes.c_int
        L.gattn_decode_int8.argtypes = [vp, vp, vp, vp, vp, vp, vp, i32, i32, ctypes.POINTER(GattnCfg), vp, sz, vp]
        L.gattn_cp_blocks.restype = ctypes.c_int
        L.gattn_cp_blocks.argtypes = [i32, i32, i32, ctypes.POINTER(i32), ctypes.POINTER(i32)]
        L.gattn_prefill_padded.restype = ctypes.c_int
        L.gattn_prefill_padded.argtypes = [vp, vp, vp, vp, vp, vp, i32, i32, ctypes.POINTER(GattnCfg), vp, sz,
                                           vp]
        _lib = L
    return _lib


def _raise_if(status: int, where: str):
    if status != GATTN_OK:
        raise GattnError(status, where, lib().gattn_last_error().decode())


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, ndim: int):
    if t.dtype != dtype or t.dim() != ndim or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected a contiguous CUDA {dtype} tensor of rank {ndim}, got "
                         f"{t.dtype} {tuple(t.shape)} on {t.device}")


@dataclass
class LayerSpec:
    """Host description of one attention layer (the fields of ``gattn_cfg``)."""
    num_heads: int
    num_kv_heads: int
    head_dim: int
    window: int = 0
    rope_theta: float = 10000.0
    rotary_fraction: float = 1.0
    rope_freq_dim: int = 0
    softcap: float = 0.0
    scalar: float = 256.0
    k_eq_v: bool = False
    qk_norm: int = NORM_NONE
    norm_eps: float = 1e-6
    keys_transformed: bool = False   # KV caches hold keys after QK-norm and RoPE

    @property
    def rot_dim(self) -> int:
        return int(round(self.rotary_fraction * self.head_dim))

    @classmethod
    def of(cls, obj) -> "LayerSpec":
        return cls(**{f: getattr(obj, f) for f in cls.__dataclass_fields__ if hasattr(obj, f)})


def rope_table(theta: float, rot_dim: int, freq_dim: int, max_pos: int, device="cuda",
               stream=None) -> torch.Tensor:
    """Device (cos, sin) table [max_pos][rot_dim/2][2] fp32 built by the library."""
    n = lib().gattn_rope_table_bytes(max_pos, rot_dim)
    if n == 0:
        raise ValueError("invalid rope table size")
    tab = torch.empty(n // 4, dtype=torch.float32, device=device)
    _raise_if(lib().gattn_rope_table_fill(_ptr(tab), theta, rot_dim, freq_dim, max_pos,
                                          _stream(stream)), "gattn_rope_table_fill")
    return tab


class AttentionLayer:
    """A layer's device-side constants (RoPE table, QK-norm gains) and its cfg."""

    def __init__(self, spec: LayerSpec, max_pos: int, w_q: Optional[torch.Tensor] = None,
                 w_k: Optional[torch.Tensor] = None, device="cuda"):
        self.spec = spec
        self.max_pos = max_pos
        R = spec.rot_dim
        F = spec.rope_freq_dim or spec.head_dim
        self.table = rope_table(spec.rope_theta, R, F, max_pos, device) if R > 0 else None
        self.w_q = None if w_q is None else w_q.to(device=device, dtype=torch.float32).contiguous()
        self.w_k = None if w_k is None else w_k.to(device=device, dtype=torch.float32).contiguous()
        self.cfg = GattnCfg(
            num_heads=spec.num_heads, num_kv_heads=spec.num_kv_heads, head_dim=spec.head_dim,
            window=spec.window, rope_theta=spec.rope_theta, rotary_fraction=spec.rotary_fraction,
            rope_freq_dim=spec.rope_freq_dim,
            rope_table=None if self.table is None else self.table.data_ptr(),
            rope_max_pos=max_pos if R > 0 else 0, softcap=spec.softcap, scalar=spec.scalar,
            k_eq_v=int(spec.k_eq_v), qk_norm=spec.qk_norm, norm_eps=spec.norm_eps,
            q_norm_w=None if self.w_q is None else self.w_q.data_ptr(),
            k_norm_w=None if self.w_k is None else self.w_k.data_ptr(),
            keys_transformed=int(spec.keys_transformed))

    # -- workspaces --------------------------------------------------------------
    def prefill_workspace(self, batch: int, seq_len: int, device="cuda") -> torch.Tensor:
        n = lib().gattn_prefill_workspace_size(ctypes.byref(self.cfg), batch, seq_len)
        if n == 0:
            raise GattnError(1, "gattn_prefill_workspace_size", "invalid cfg or sizes")
        ws = torch.empty(n, dtype=torch.uint8, device=device)
        _raise_if(lib().gattn_workspace_init(_ptr(ws), n, _stream()), "gattn_workspace_init")
        return ws

    def decode_workspace(self, batch: int, max_len: int, device="cuda") -> torch.Tensor:
        n = lib().gattn_decode_workspace_size(ctypes.byref(self.cfg), batch, max_len)
        if n == 0:
            raise GattnError(1, "gattn_decode_workspace_size", "invalid cfg or sizes")
        ws = torch.empty(n, dtype=torch.uint8, device=device)
        _raise_if(lib().gattn_workspace_init(_ptr(ws), n, _stream()), "gattn_workspace_init")
        return ws

    # -- the two entry points ---------------------------------------------------
    def prefill(self, q, k, v=None, positions=None, out=None, workspace=None, stream=None, seq_range=None):
        """gattn_prefill: q [B,S,H,D], k/v [B,S,Hkv,D] bf16, positions [B,S] int32.

        With ``seq_range`` (int32 [B,2], sequence b's valid tokens [lo, hi)) this calls
        gattn_prefill_padded: padding tokens are neither queries nor keys, their rows are zero."""
        _need(q, "q", torch.bfloat16, 4)
        _need(k, "k", torch.bfloat16, 4)
        if v is not None:
            _need(v, "v", torch.bfloat16, 4)
        B, S = q.shape[0], q.shape[1]
        if positions is None and self.spec.rot_dim > 0:
            raise ValueError("positions are required when RoPE is on")
        if positions is not None:
            _need(positions, "positions", torch.int32, 2)
        out = torch.empty_like(q) if out is None else out
        ws = self.prefill_workspace(B, S, q.device) if workspace is None else workspace
        if seq_range is not None:
            _need(seq_range, "seq_range", torch.int32, 2)
            if tuple(seq_range.shape) != (B, 2):
                raise ValueError(f"seq_range must be [{B}, 2], got {tuple(seq_range.shape)}")
            _raise_if(lib().gattn_prefill_padded(_ptr(q), _ptr(k), _ptr(v), _ptr(positions), _ptr(seq_range),
                                                 _ptr(out), B, S, ctypes.byref(self.cfg), _ptr(ws), ws.numel(),
                                                 _stream(stream)),
                      "gattn_prefill_padded")
            return out
        _raise_if(lib().gattn_prefill(_ptr(q), _ptr(k), _ptr(v), _ptr(positions), _ptr(out), B, S,
                                      ctypes.byref(self.cfg), _ptr(ws), ws.numel(), _stream(stream)),
                  "gattn_prefill")
        return out

    def decode(self, q, k_cache, v_cache=None, seq_lens=None, out=None, workspace=None, stream=None):
        """gattn_decode: q [B,H,D], caches [B,Lmax,Hkv,D] bf16 (raw keys/values), seq_lens [B] int32."""
        _need(q, "q", torch.bfloat16, 3)
        _need(k_cache, "k_cache", torch.bfloat16, 4)
        if v_cache is not None:
            _need(v_cache, "v_cache", torch.bfloat16, 4)
        _need(seq_lens, "seq_lens", torch.int32, 1)
        B, Lmax = k_cache.shape[0], k_cache.shape[1]
        out = torch.empty_like(q) if out is None else out
        ws = self.decode_workspace(B, Lmax, q.device) if workspace is None else workspace
        _raise_if(lib().gattn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), _ptr(out),
                                     B, Lmax, ctypes.byref(self.cfg), _ptr(ws), ws.numel(),
                                     _stream(stream)), "gattn_decode")
        return out


    def prefill_chunk_workspace(self, batch: int, chunk_len: int, max_len: int, device="cuda") -> torch.Tensor:
        n = lib().gattn_prefill_chunk_workspace_size(ctypes.byref(self.cfg), batch, chunk_len, max_len)
        if n == 0:
            raise GattnError(1, "gattn_prefill_chunk_workspace_size", "invalid cfg or sizes")
        ws = torch.empty(n, dtype=torch.uint8, device=device)
        _raise_if(lib().gattn_workspace_init(_ptr(ws), n, _stream()), "gattn_workspace_init")
        return ws

    def prefill_chunk(self, q, k_cache, v_cache=None, prefix_lens=None, k_new=None, v_new=None, out=None,
                      workspace=None, stream=None):
        """gattn_prefill_chunk: q [B,C,H,D] at positions prefix_lens[b] + i against caches
        [B,Lmax,Hkv,D] (raw keys/values); k_new/v_new [B,C,Hkv,D] are appended first when given."""
        _need(q, "q", torch.bfloat16, 4)
        _need(k_cache, "k_cache", torch.bfloat16, 4)
        if v_cache is not None:
            _need(v_cache, "v_cache", torch.bfloat16, 4)
        for t, n in ((k_new, "k_new"), (v_new, "v_new")):
            if t is not None:
                _need(t, n, torch.bfloat16, 4)
        _need(prefix_lens, "prefix_lens", torch.int32, 1)
        B, C = q.shape[0], q.shape[1]
        Lmax = k_cache.shape[1]
        out = torch.empty_like(q) if out is None else out
        ws = self.prefill_chunk_workspace(B, C, Lmax, q.device) if workspace is None else workspace
        _raise_if(lib().gattn_prefill_chunk(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                            _ptr(prefix_lens), _ptr(out), B, C, Lmax, ctypes.byref(self.cfg),
                                            _ptr(ws), ws.numel(), _stream(stream)), "gattn_prefill_chunk")
        return out

    def kv_append(self, k_new, v_new, k_cache, v_cache, cache_lens, status=None, stream=None):
        """gattn_kv_append_layer: rows [B,n,Hkv,D] into caches [B,Lmax,Hkv,D] at rows
        [cache_lens[b], +n); keys written transformed when the spec's keys_transformed is set."""
        _need(k_new, "k_new", torch.bfloat16, 4)
        _need(k_cache, "k_cache", torch.bfloat16, 4)
        if v_new is not None:
            _need(v_new, "v_new", torch.bfloat16, 4)
            _need(v_cache, "v_cache", torch.bfloat16, 4)
        _need(cache_lens, "cache_lens", torch.int32, 1)
        B, n = k_new.shape[0], k_new.shape[1]
        _raise_if(lib().gattn_kv_append_layer(ctypes.byref(self.cfg), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                              _ptr(v_cache), _ptr(cache_lens), B, n, k_cache.shape[1], _ptr(status),
                                              _stream(stream)), "gattn_kv_append_layer")

    def decode_int8(self, q, k_codes, k_scales, v_codes=None, v_scales=None, seq_lens=None, out=None,
                    workspace=None, stream=None):
        """gattn_decode_int8: q [B,H,D] bf16; codes [B,Lmax,Hkv,D] int8 and scales [B,Lmax,Hkv] fp32
        (from ``kv_quantize``) of the raw keys/values; seq_lens [B] int32."""
        _need(q, "q", torch.bfloat16, 3)
        _need(k_codes, "k_codes", torch.int8, 4)
        _need(k_scales, "k_scales", torch.float32, 3)
        if v_codes is not None:
            _need(v_codes, "v_codes", torch.int8, 4)
            _need(v_scales, "v_scales", torch.float32, 3)
        _need(seq_lens, "seq_lens", torch.int32, 1)
        B, Lmax = k_codes.shape[0], k_codes.shape[1]
        if tuple(k_scales.shape) != tuple(k_codes.shape[:3]):
            raise ValueError("k_scales must be [B, Lmax, Hkv]")
        if v_codes is not None and tuple(v_scales.shape) != tuple(v_codes.shape[:3]):
            raise ValueError("v_scales must be [B, Lmax, Hkv]")
        out = torch.empty_like(q) if out is None else out
        ws = self.decode_workspace(B, Lmax, q.device) if workspace is None else workspace
        _raise_if(lib().gattn_decode_int8(_ptr(q), _ptr(k_codes), _ptr(k_scales), _ptr(v_codes), _ptr(v_scales),
                                          _ptr(seq_lens), _ptr(out), B, Lmax, ctypes.byref(self.cfg), _ptr(ws),
                                          ws.numel(), _stream(stream)), "gattn_decode_int8")
        return out


def kv_append(k_new, v_new, k_cache, v_cache, cache_lens, status=None, stream=None):
    """gattn_kv_append: rows [B,n,Hkv,D] into caches [B,Lmax,Hkv,D] at rows [cache_lens[b], +n)."""
    _need(k_new, "k_new", torch.bfloat16, 4)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    if v_new is not None:
        _need(v_new, "v_new", torch.bfloat16, 4)
        _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(cache_lens, "cache_lens", torch.int32, 1)
    B, n, Hkv, D = k_new.shape
    _raise_if(lib().gattn_kv_append(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(cache_lens), B, n,
                                    k_cache.shape[1], Hkv, D, _ptr(status), _stream(stream)), "gattn_kv_append")


def kv_quantize(x: torch.Tensor, codes=None, scales=None, stream=None):
    """gattn_kv_quantize: x [..., D] bf16 -> (codes [..., D] int8, scales [...] fp32)."""
    if x.dtype != torch.bfloat16 or not x.is_cuda or not x.is_contiguous() or x.dim() < 1:
        raise ValueError("x: expected a contiguous CUDA bfloat16 tensor")
    D = x.shape[-1]
    codes = torch.empty(x.shape, dtype=torch.int8, device=x.device) if codes is None else codes
    scales = torch.empty(x.shape[:-1], dtype=torch.float32, device=x.device) if scales is None else scales
    _raise_if(lib().gattn_kv_quantize(_ptr(x), _ptr(codes), _ptr(scales), x.numel() // max(D, 1), D,
                                      _stream(stream)), "gattn_kv_quantize")
    return codes, scales


def decode_noalloc(layer: "AttentionLayer", q, k_cache, v_cache=None, seq_lens=None, out=None,
                   stream=None):
    """gattn_decode_noalloc: the decode step without a workspace (library-held scratch)."""
    _need(q, "q", torch.bfloat16, 3)
    _need(k_cache, "k_cache", torch.bfloat16, 4)
    if v_cache is not None:
        _need(v_cache, "v_cache", torch.bfloat16, 4)
    _need(seq_lens, "seq_lens", torch.int32, 1)
    B, Lmax = k_cache.shape[0], k_cache.shape[1]
    out = torch.empty_like(q) if out is None else out
    _raise_if(lib().gattn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(seq_lens), _ptr(out),
                                         B, Lmax, ctypes.byref(layer.cfg), _stream(stream)),
              "gattn_decode_noalloc")
    return out


def check(workspace: torch.Tensor, stream=None) -> int:
    """gattn_check: synchronise, read and clear the status word; returns the status code."""
    return lib().gattn_check(_stream(stream), _ptr(workspace))


def selftest_wait_timeout(workspace: torch.Tensor, timeout_us: int, stream=None):
    _raise_if(lib().gattn_selftest_wait_timeout(_ptr(workspace), workspace.numel(), timeout_us,
                                                _stream(stream)), "gattn_selftest_wait_timeout")


def set_wait_timeout_us(us: int):
    lib().gattn_set_wait_timeout_us(us)


def set_profile_events(start=None, stop=None):
    """Time the main kernel of later calls: ``start``/``stop`` are torch.cuda.Event (or None)."""
    lib().gattn_set_profile_events(None if start is None else ctypes.c_void_p(start.cuda_event),
                                   None if stop is None else ctypes.c_void_p(stop.cuda_event))


def set_trace_buffer(buf: Optional[torch.Tensor] = None):
    """Record per-CTA prefill timelines into ``buf`` (int64 CUDA tensor), or stop (None)."""
    if buf is None:
        lib().gattn_set_trace_buffer(None, 0)
    else:
        lib().gattn_set_trace_buffer(ctypes.c_void_p(buf.data_ptr()), buf.numel() * buf.element_size())


def version() -> str:
    return lib().gattn_version().decode()


def cp_blocks(seq_len: int, world: int, rank: int):
    """gattn_cp_blocks: rank's two token blocks [(start, len), (start, len)] of a prompt of
    seq_len tokens split over `world` ranks (zig-zag: blocks rank and 2*world-1-rank of 2*world)."""
    starts = (ctypes.c_int32 * 2)()
    lens = (ctypes.c_int32 * 2)()
    _raise_if(lib().gattn_cp_blocks(seq_len, world, rank, starts, lens), "gattn_cp_blocks")
    return [(int(starts[0]), int(lens[0])), (int(starts[1]), int(lens[1]))]
