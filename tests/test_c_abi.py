"""The library used from plain C: tests/c_abi/consumer.c includes only include/dsa.h (and the
CUDA runtime for its own device memory), is compiled with gcc as C99 with every warning an
error, and links libdsa.so directly.  On the CPU it runs the host-side checks (status strings,
argument validation); on a GPU it also runs a top-k against a brute-force selection written in
C and reads the bounded-wait self-test's DSA_ERR_TIMEOUT through dsa_device_error."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    import sparse_attention_09_b200 as dsa
    lib_dir = os.path.dirname(dsa.lib_path())
    gcc = shutil.which("gcc")
    assert gcc, "gcc not found"
    exe = str(tmp_path / "dsa_consumer")
    cmd = [gcc, "-std=c99", "-Wall", "-Wextra", "-Werror",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.join(ROOT, "tests", "c_abi", "consumer.c"),
           "-L", lib_dir, "-ldsa", f"-Wl,-rpath,{lib_dir}",
           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}",
           "-o", exe]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    return exe


def test_c_consumer_compiles_and_passes_host_checks(tmp_path):
    exe = _build(tmp_path)
    res = subprocess.run([exe, "host"], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "dsa C consumer: ok (host checks)" in res.stdout


@pytest.mark.gpu
def test_c_consumer_device_checks(tmp_path):
    exe = _build(tmp_path)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "dsa C consumer: ok (host and device checks)" in res.stdout
