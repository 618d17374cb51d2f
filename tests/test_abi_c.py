"""The C ABI from C: include/gattn.h compiles as plain C99, a C program linked against
libgattn.so sees the gattn_cfg layout the Python mirror has, and the library answers
its host-side calls from C (status strings, sizes, argument validation; no launch)."""
import ctypes
import os
import shutil
import subprocess

import pytest

import gemma_family_decoder_b200 as G
from gemma_family_decoder_b200 import gattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "abi_check.c")

pytestmark = pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")


def test_header_is_plain_c99():
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-fsyntax-only", "-x", "c",
                        os.path.join(ROOT, "include", "gattn.h")], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_c_client_layout_and_host_calls(tmp_path):
    G.lib()  # builds nothing: the library must exist already
    exe = tmp_path / "abi_check"
    libdir = os.path.dirname(gattn.LIB_PATH)
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), SRC, "-o",
                        str(exe), "-L", libdir, "-lgattn", f"-Wl,-rpath,{libdir}"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stderr
    out = dict(line.split("=", 1) for line in run.stdout.strip().splitlines())
    assert int(out["sizeof"]) == ctypes.sizeof(G.GattnCfg)
    for field in ("rope_table", "q_norm_w", "keys_transformed"):
        assert int(out[f"offset {field}"]) == getattr(G.GattnCfg, field).offset, field
    assert out["version"] == gattn.lib().gattn_version().decode()
    assert out["status6"] == gattn.lib().gattn_status_string(6).decode()
    assert int(out["rope_bytes"]) == 100 * 64 * 8 and int(out["rope_bytes_bad"]) == 0
    assert int(out["prefill_ws"]) == G.lib().gattn_prefill_workspace_size(
        ctypes.byref(G.GattnCfg(num_heads=8, num_kv_heads=1, head_dim=256, rope_theta=1e4, scalar=256.0,
                                norm_eps=1e-6)), 2, 300)
    assert int(out["decode_ws"]) > 0
    assert int(out["prefill_null_q"]) == 1 and out["last_error_set"] == "1"
    assert int(out["decode_d128"]) == 2
    assert int(out["decode_kt_keqv"]) == 1
    assert int(out["prefill_empty"]) == 0
    assert int(out["quantize_d100"]) == 2
