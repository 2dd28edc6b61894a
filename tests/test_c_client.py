"""The C ABI from plain C: tests/c_abi_client.c is compiled as C99 with -pedantic
-Werror against include/sla.h, linked against libsla.so and run (host-side entry
points only; no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import block_sparse_linear_sm_b200 as sla

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_client_compiles_links_and_runs():
    lib = sla.lib()  # builds nothing; fails loudly if libsla.so is missing
    libdir = os.path.dirname(lib._name)
    out_dir = os.path.join(ROOT, "_build")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "c_abi_client")
    cmd = ["gcc", "-std=c99", "-pedantic", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), os.path.join(HERE, "c_abi_client.c"),
           "-L", libdir, "-l:libsla.so", f"-Wl,-rpath,{libdir}", "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
