"""The public header compiles as plain C99 (-Wall -Wextra -Werror) and a C
program drives libpa.so's host-side calls through the C ABI (no GPU)."""
import os
import shutil
import subprocess

import pytest

import paged_kv_attention_token_b200 as pa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c99_client_against_the_library(tmp_path):
    from paged_kv_attention_token_b200 import build
    lib = build.build()
    exe = tmp_path / "pa_c_client"
    libdir = os.path.dirname(lib)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "pa_c_client.c"), "-o", str(exe),
           f"-L{libdir}", f"-Wl,-rpath,{libdir}", "-l:" + os.path.basename(lib)]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr + r.stdout
    assert "C client ok" in r.stdout
