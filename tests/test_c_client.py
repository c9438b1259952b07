"""The C ABI from plain C: tests/c/abi_host.c compiles as C99 against
include/moe.h, links libmoe_b200.so and exercises the host-side entry points
(no GPU work)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_plain_c_client(tmp_path):
    from mixture_experts_layer_sqrt_b200 import build
    lib = build.build()
    exe = tmp_path / "abi_host"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host.c"), lib, "-o", str(exe),
                    "-Wl,-rpath," + os.path.dirname(lib)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    assert "abi_host: ok" in r.stdout
