"""The library from plain C: tests/c/abi_consumer.c is compiled with gcc
against include/flowcache.h and linked with libflowcache.so and the CUDA
runtime, then run (host checks here; the hand-worked gate trace on a GPU)."""

import os
import shutil
import subprocess

import pytest

import cache_gating_kv_b200 as fc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


@pytest.fixture(scope="module")
def consumer(tmp_path_factory):
    if shutil.which("gcc") is None:
        pytest.skip("gcc is not installed")
    fc.library()  # builds nothing; fails loudly if the library is missing
    libdir = os.path.dirname(fc.library_path)
    exe = str(tmp_path_factory.mktemp("c") / "abi_consumer")
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Werror", "-o", exe,
           os.path.join(ROOT, "tests", "c", "abi_consumer.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", libdir, "-lflowcache", "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + libdir + ":" + os.path.join(CUDA, "lib64")]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_consumer_host_checks(consumer):
    out = subprocess.run([consumer], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"


@pytest.mark.gpu
def test_c_consumer_gate_trace_on_gpu(consumer):
    out = subprocess.run([consumer, "gpu"], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
