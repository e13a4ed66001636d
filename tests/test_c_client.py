"""The C ABI from a plain C program: include/relkl.h compiles as C11 with gcc,
the program links against the in-tree librelkl.so, and argument validation,
status strings and path selection behave as the header states (no GPU)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "attention_relation_kl_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_client(tmp_path):
    lib = os.path.join(LIBDIR, "librelkl.so")
    if not os.path.exists(lib):
        pytest.skip("librelkl.so not built")
    exe = str(tmp_path / "abi_check")
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), os.path.join(ROOT, "tests", "c", "abi_check.c"),
           "-L", LIBDIR, "-lrelkl", f"-Wl,-rpath,{LIBDIR}", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    env = dict(os.environ)
    cuda_lib = "/usr/local/cuda/lib64"
    env["LD_LIBRARY_PATH"] = cuda_lib + (":" + env["LD_LIBRARY_PATH"] if env.get("LD_LIBRARY_PATH") else "")
    res = subprocess.run([exe], capture_output=True, text=True, env=env, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    assert res.stdout.strip().startswith("ok "), res.stdout
