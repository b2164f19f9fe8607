"""The C ABI is usable from plain C: tests/c_consumer.c includes only
include/diffattn.h, compiles as C99 with warnings as errors, links
libdiffattn.so and checks the host-side contract (validation codes,
workspace formulas, declared signatures) without a GPU."""
import os
import shutil
import subprocess

import pytest

from differential_attention_04_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _cuda_include():
    for cand in (os.environ.get("CUDA_HOME"), "/usr/local/cuda"):
        if cand and os.path.exists(os.path.join(cand, "include", "cuda_runtime_api.h")):
            return os.path.join(cand, "include")
    return None


def test_c_consumer(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    inc = _cuda_include()
    if cc is None or inc is None:
        pytest.skip("no C compiler or CUDA headers")
    lib = build()
    libdir = os.path.dirname(lib)
    exe = str(tmp_path / "c_consumer")
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", inc,
           os.path.join(ROOT, "tests", "c_consumer.c"), "-o", exe, "-L", libdir, "-ldiffattn",
           f"-Wl,-rpath,{libdir}"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "c consumer ok" in r.stdout, r.stdout + r.stderr
