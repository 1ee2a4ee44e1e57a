"""The C ABI used from plain C: tests/c/abi_host_check.c is compiled as C11
against include/kvq.h, linked to libkvq.so and run (host-side entry points
only, no GPU needed)."""
import os
import subprocess

import pytest

from long_context_decode_dual_b200 import kvq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA_LIB = "/usr/local/cuda/lib64"


def test_c_program_uses_the_abi(tmp_path):
    lib = kvq.LIB_PATH
    if not os.path.exists(lib):
        pytest.skip("libkvq.so not built")
    exe = tmp_path / "abi_host_check"
    libdir = os.path.dirname(lib)
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "abi_host_check.c"), "-o", str(exe),
                           "-L", libdir, "-lkvq", f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{CUDA_LIB}"])
    out = subprocess.run([str(exe)], capture_output=True, text=True, check=True).stdout.splitlines()
    got = dict(line.split(" ", 1) for line in out)
    assert got["version"] == str(kvq.lib().kvq_version())
    assert got["page_bytes"] == "12544 20736 9472 0"
    assert got["num_selected"] == "128 77 52 -1"
    assert got["status_words"] == str(1 + 2 + 16)
    assert got["cache_bytes"] == str(2 * 8 * 2 * 12544)
    assert got["cache_bytes_tier"] == str(2 * 8 * (2 * 9472 + 320 * 512))
    assert got["num_buckets"] == "2"
    assert got["append_null"] == "-1" and got["init_null"] == "-1" and got["copy_null"] == "-1"
    assert got["string"] == "capacity exceeded"
