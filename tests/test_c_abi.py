"""The C ABI from plain C: tests/c_abi_smoke.c includes only include/hs2.h,
is compiled with gcc and linked against the in-tree libhs2.so, and calls the
entry points that launch nothing (size queries, argument checks)."""
import os
import shutil
import subprocess

import pytest

from token_level_sparse_causal_b200 import hs2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_uses_the_header_and_library(tmp_path):
    hs2.lib()  # the library is built in-tree
    libdir = os.path.dirname(hs2.LIB_PATH)
    exe = tmp_path / "c_abi_smoke"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_smoke.c"), "-o", str(exe), f"-L{libdir}", "-l:libhs2.so",
                    f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout
    got = dict(line.split(" ", 1) for line in out.strip().splitlines())
    L, Hkv = 131072, 8
    assert got["full_ws_rc"] == "0"
    assert int(got["full_ws_bytes"]) >= Hkv * (L - 128) * 4
    assert got["fa_ws_rc"] == "0" and got["fa_ws_bytes_bf16"] == "0"
    assert int(got["fa_ws_bytes_e4m3"]) >= 2 * L * Hkv * 128 * 2
    assert got["decode_ws_rc"] == "0" and int(got["decode_ws_bytes"]) > 0
    assert int(got["bad_d_rc"]) == hs2.HS2_ERR_UNSUPPORTED
    assert int(got["version"]) >= 100
    assert "timed out" in got["strerror_timeout"]
