"""The boundary from plain C: include/eqlin.h compiles as C99 with -pedantic and no
warnings, and a C program linked against libeqlin.so calls the host-only entry points
(no GPU needed)."""
from __future__ import annotations

import os
import shutil
import subprocess

import pytest

import cyclic_group_dft_b200 as eq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_links(tmp_path):
    lib_dir = os.path.dirname(eq._capi.LIB_PATH)
    exe = tmp_path / "c_abi_check"
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c_abi_check.c"),
           "-L", lib_dir, "-leqlin", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.strip()
    fields = dict(kv.split("=", 1) for kv in out.split(" ", 7))
    assert fields["query"] == "0" and fields["path"] == "0"          # tokens on N, resident weights
    assert fields["dw_query"] == "0" and fields["dw_tokens"] == "16"
    assert int(fields["odd_g"]) == eq.EQLIN_ERR_UNSUPPORTED
    assert int(fields["null_forward"]) == eq.EQLIN_ERR_INVALID_ARG
    assert int(fields["version"]) > 0 and "timed out" in fields["timeout_text"]
