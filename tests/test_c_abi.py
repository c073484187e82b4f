"""The boundary from C: tests/c_abi_check.c includes only include/lkv.h, is compiled with gcc and
linked against liblkv.so, and checks the host-only entry points (no GPU, no CUDA call)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "latent_kv_cache_split_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc is not installed")
def test_plain_c_program_uses_the_library():
    import importlib.util
    spec = importlib.util.spec_from_file_location("lkv_build", os.path.join(PKG, "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build()
    out_dir = os.path.join(ROOT, "tests", "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "c_abi_check")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c_abi_check.c"), "-L", PKG, "-llkv",
                    f"-Wl,-rpath,{PKG}", "-o", exe], check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
