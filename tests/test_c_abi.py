"""The boundary used from C: tests/c/abi_host_check.c is compiled with gcc against include/vdn.h,
linked with libvdn.so and run; it calls only host-side entry points (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
LIBDIR = os.path.join(ROOT, "video_diffusion_linear_b200")


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_c_caller(tmp_path):
    from video_diffusion_linear_b200 import build
    build.build()
    exe = tmp_path / "abi_host_check"
    cuda_lib = "/usr/local/cuda/lib64"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host_check.c"), "-L", LIBDIR, "-lvdn",
                    "-Wl,-rpath," + LIBDIR, "-o", str(exe)], check=True)
    env = dict(os.environ)
    env["LD_LIBRARY_PATH"] = ":".join(p for p in (LIBDIR, cuda_lib, env.get("LD_LIBRARY_PATH", "")) if p)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True, env=env).stdout.split("\n")
    assert out[0] == "bounds 0 5 19"
    assert out[1] == "bounds_bad_chunk 1"                 # VDN_ERR_INVALID_ARG
    assert out[2] == "sizes 1 1 1 256"
    assert out[3] == "unsupported 1"
    assert out[4].startswith("null_q 1 ")                 # validation error, before any launch
    assert out[5] == "frames 0:0-15 0:15-25 0:25-31 owner 0 2"
    assert out[6] == "map_bytes 1"
