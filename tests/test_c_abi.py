"""The C ABI from plain C: tests/c/abi_host_check.c includes include/attn.h as C99 (no C++
constructs may leak into the header), links the built library and calls its host-only
entry points (tile classes, dry-run plan, error statuses). No GPU is needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_header_compiles_as_c_and_host_calls_work(attn_lib, tmp_path):
    lib_dir = os.path.dirname(attn_lib._LIB_PATH)
    exe = str(tmp_path / "abi_host_check")
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host_check.c"), "-o", exe, "-L", lib_dir, "-lattn_b200",
           f"-Wl,-rpath,{lib_dir}"]
    build = subprocess.run(cmd, capture_output=True, text=True)
    assert build.returncode == 0, build.stderr
    run = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0 and run.stdout.strip() == "ok", run.stdout + run.stderr
