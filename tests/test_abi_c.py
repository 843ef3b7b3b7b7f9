"""The C ABI used from C: tests/c/abi_from_c.c is compiled with gcc against
include/fa_b200.h, linked with the library and run (no GPU needed: every call
it makes answers during argument validation or host-side arithmetic)."""
import os
import shutil
import subprocess

import pytest

from exact_attention_forward_flash_b200 import build as fa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_calls_the_abi(tmp_path):
    lib = fa_build.build()
    exe = tmp_path / "abi_from_c"
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "abi_from_c.c"), "-o", str(exe),
                           lib, "-Wl,-rpath," + os.path.dirname(lib)])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == "ok"
