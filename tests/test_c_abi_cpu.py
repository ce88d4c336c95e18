"""The C ABI from plain C: tests/c_abi/abi_check.c is compiled with gcc as C11 against
include/libgdn.h, linked against the built libgdn.so and run (no GPU needed: it exercises
only calls that enqueue nothing)."""
import os
import shutil
import subprocess

import pytest

from linear_attention_recurrence_05_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_INC = "/usr/local/cuda/include"


@pytest.mark.skipif(shutil.which("gcc") is None or not os.path.isdir(CUDA_INC),
                    reason="needs gcc and the CUDA runtime headers")
def test_c_client_compiles_links_and_runs():
    lib = _native.LIB_PATH
    assert os.path.exists(lib), "build libgdn.so first"
    out = os.path.join(ROOT, "tests", "c_abi", "_build")
    os.makedirs(out, exist_ok=True)
    exe = os.path.join(out, f"abi_check.{os.getpid()}")
    cmd = ["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", f"-I{ROOT}/include", f"-I{CUDA_INC}",
           os.path.join(ROOT, "tests", "c_abi", "abi_check.c"), "-o", str(exe),
           f"-L{os.path.dirname(lib)}", "-l:libgdn.so", f"-Wl,-rpath,{os.path.dirname(lib)}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    try:
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    finally:
        os.remove(exe)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "libgdn C ABI ok" in r.stdout
    # the binding's copy of the no-allocation scratch limit is the header's value
    line = [ln for ln in r.stdout.splitlines() if ln.startswith("GDN_STATIC_SCRATCH_BYTES")]
    assert line and int(line[0].split()[1]) == _native.STATIC_SCRATCH_BYTES
