"""The C ABI from C.

tests/c/abi_consumer.c includes only include/paged_kv.h.  It must compile as
C99 with every warning an error, link against libpaged_kv.so, and pass its
checks.  Host mode runs here.  GPU mode needs a B200: it runs a copy + write +
decode step through the C ABI on cudaMalloc'd buffers and checks it against
the oracle library.
"""

import os
import subprocess

import pytest

from tests.conftest import ROOT

PKG = os.path.join(ROOT, "paged_kv_cache_398_b200")
SRC = os.path.join(ROOT, "tests", "c", "abi_consumer.c")
CUDA = "/usr/local/cuda"


def _compile(tmp_path, gpu: bool) -> str:
    from paged_kv_cache_398_b200.build import build_library
    build_library()
    exe = str(tmp_path / ("abi_consumer_gpu" if gpu else "abi_consumer"))
    cmd = ["gcc", "-std=c99", "-O1", "-Wall", "-Wextra", "-Werror", "-pedantic",
           "-I", os.path.join(ROOT, "include"), SRC, "-o", exe,
           "-L", PKG, "-lpaged_kv", f"-Wl,-rpath,{PKG}"]
    if gpu:
        import oracle
        odir = os.path.dirname(oracle.build_oracle())
        cmd += ["-DWITH_CUDA", "-isystem", f"{CUDA}/include", "-L", odir, "-loracle", f"-Wl,-rpath,{odir}",
                "-L", f"{CUDA}/lib64", "-lcudart", f"-Wl,-rpath,{CUDA}/lib64"]
    cmd += ["-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    return exe


def _run(exe: str, mode: str):
    r = subprocess.run([exe, mode], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr


def test_header_compiles_as_c99_and_host_calls_work(tmp_path):
    _run(_compile(tmp_path, gpu=False), "host")


def test_gpu_consumer_builds(tmp_path):
    _compile(tmp_path, gpu=True)


@pytest.mark.gpu
def test_decode_step_from_c_matches_the_oracle(tmp_path):
    _run(_compile(tmp_path, gpu=True), "gpu")
