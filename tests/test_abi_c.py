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


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not installed")
def test_c_program_runs_a_forward_that_matches_the_oracle(tmp_path):
    import numpy as np
    import torch

    import fa_inputs
    import oracle
    from parity_util import compare

    lib = fa_build.build()
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    exe = tmp_path / "fwd_from_c"
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(cuda, "include"),
                           os.path.join(ROOT, "tests", "c", "fwd_from_c.c"), "-o", str(exe),
                           lib, "-Wl,-rpath," + os.path.dirname(lib),
                           "-L", os.path.join(cuda, "lib64"), "-lcudart",
                           "-Wl,-rpath," + os.path.join(cuda, "lib64")])
    B, Sq, Sk, Hq, Hkv, D = 2, 200, 333, 8, 2, 128
    p = fa_inputs.random_dense(1500, B, Sq, Sk, Hq, Hkv, D, causal=True)
    raw = torch.cat([p.q.reshape(-1), p.k.reshape(-1), p.v.reshape(-1)]).view(torch.int16)
    (tmp_path / "in.bin").write_bytes(raw.numpy().tobytes())
    r = subprocess.run([str(exe), str(tmp_path / "in.bin"), str(tmp_path / "out.bin"),
                        *map(str, (B, Sq, Sk, Hq, Hkv, D, 1))],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr
    data = (tmp_path / "out.bin").read_bytes()
    no = B * Sq * Hq * D
    o = torch.frombuffer(bytearray(data[:2 * no]), dtype=torch.bfloat16).reshape(B, Sq, Hq, D)
    lse = np.frombuffer(data[2 * no:], dtype=np.float32).reshape(B, Hq, Sq)
    ro, rl = oracle.attention(p.q, p.k, p.v, causal=True, softmax_scale=p.softmax_scale)
    compare(o, lse, ro, rl, what="forward from C")
