"""include/moe.h used from plain C: tests/c/abi_host.c compiles as C99 with
gcc (-Wall -Wextra -Werror -pedantic) against the header, links libmoe and
runs. The CPU test runs its host-only checks; the GPU test adds a context on
device 0."""
import os
import shutil
import subprocess

import pytest

from bit_expert_ffn_router_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "abi_host.c")


def _compile(tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not found")
    B.build()
    exe = str(tmp_path / "abi_host")
    libdir = os.path.dirname(B.LIB)
    cmd = ["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
           SRC, "-o", exe, "-L", libdir, "-lmoe", "-Wl,-rpath," + libdir]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    return exe


def test_plain_c_client_host_calls(tmp_path):
    exe = _compile(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr


@pytest.mark.gpu
def test_plain_c_client_with_a_context(tmp_path):
    exe = _compile(tmp_path)
    r = subprocess.run([exe, "gpu"], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
