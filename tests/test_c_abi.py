"""The C ABI consumed from plain C (tests/c/abi_consumer.c), without Python in between."""
import os
import subprocess

import pytest

import video_vae_convolution_implicit_b200 as c3

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "c", "abi_consumer.c")
LIBDIR = os.path.dirname(c3.lib_path)


def _run(exe, mode):
    env = dict(os.environ, LD_LIBRARY_PATH=LIBDIR + ":" + os.environ.get("LD_LIBRARY_PATH", ""))
    return subprocess.run([exe, mode], capture_output=True, text=True, env=env, timeout=300)


def test_c_consumer_cpu_checks(tmp_path):
    exe = str(tmp_path / "abi_consumer")
    subprocess.run(["gcc", "-std=c11", "-O1", "-I", os.path.join(ROOT, "include"), SRC, "-o", exe,
                    "-L", LIBDIR, "-lconv3d", "-Wl,-rpath," + LIBDIR], check=True)
    r = _run(exe, "cpu")
    assert r.returncode == 0, r.stderr


@pytest.mark.gpu
def test_c_consumer_gpu_centre_delta(tmp_path):
    exe = str(tmp_path / "abi_consumer_gpu")
    subprocess.run(["nvcc", "-Wno-deprecated-gpu-targets", "-x", "c", "-DABI_CONSUMER_GPU", "-I", os.path.join(ROOT, "include"),
                    SRC, "-o", exe, "-L", LIBDIR, "-lconv3d", "-Xlinker", "-rpath=" + LIBDIR],
                   check=True)
    r = _run(exe, "gpu")
    assert r.returncode == 0, r.stderr
