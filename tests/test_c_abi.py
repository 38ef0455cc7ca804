"""The C ABI from plain C: tests/c_abi/ea_c_smoke.c includes include/ea.h as a
C99 translation unit, links libea.so and the CUDA runtime, and drives the
router and the fused prefill with no Python on its path.  On the CPU the
program must compile and link; on a GPU its output must match the oracle."""
import os
import shutil
import subprocess

import numpy as np
import pytest

from sparse_attention_head_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c_abi", "ea_c_smoke.c")
CUDA = "/usr/local/cuda"


def _compile(out_dir):
    build.build()
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    lib_dir = os.path.dirname(build.LIB)
    exe = os.path.join(out_dir, "ea_c_smoke")
    cmd = [cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-O1",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"), SRC,
           "-o", exe, "-L", lib_dir, "-l:libea.so", "-L", os.path.join(CUDA, "lib64"),
           "-lcudart", f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stdout + res.stderr
    return exe


def test_header_and_program_compile_as_c(tmp_path):
    exe = _compile(str(tmp_path))
    assert os.path.exists(exe)


@pytest.mark.gpu
def test_c_program_matches_oracle(tmp_path):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    from gpu_common import compare
    exe = _compile(str(tmp_path))
    dump = os.path.join(str(tmp_path), "dump.bin")
    res = subprocess.run([exe, dump], capture_output=True, text=True, timeout=300)
    assert res.returncode == 0, res.stdout + res.stderr
    raw = open(dump, "rb").read()
    B, Hq, Hkv, N, d, S, W, hidden, ver = np.frombuffer(raw[:36], dtype=np.int32)
    assert ver >> 16 == 1
    pos = 36

    def take(dtype, count):
        nonlocal pos
        a = np.frombuffer(raw, dtype=dtype, count=count, offset=pos)
        pos += a.nbytes
        return a

    def bf16(a):
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)

    q = bf16(take(np.uint16, B * Hq * N * d)).reshape(B, Hq, N, d)
    k = bf16(take(np.uint16, B * Hkv * N * d)).reshape(B, Hkv, N, d)
    v = bf16(take(np.uint16, B * Hkv * N * d)).reshape(B, Hkv, N, d)
    w1 = take(np.float32, hidden * Hkv * d).reshape(hidden, Hkv * d).astype(np.float64)
    b1 = take(np.float32, hidden).astype(np.float64)
    w2 = take(np.float32, Hq * hidden).reshape(Hq, hidden).astype(np.float64)
    b2 = take(np.float32, Hq).astype(np.float64)
    mask = take(np.uint8, B * Hq).reshape(B, Hq)
    out = bf16(take(np.uint16, B * Hq * N * d)).reshape(B, Hq, N, d)
    assert pos == len(raw)
    ref_mask, _ = oracle.router_decide(k, w1, b1, w2, b2)
    np.testing.assert_array_equal(mask, ref_mask)
    assert mask.tolist() == [[0, 1, 1, 0]]
    ref = oracle.attention(q, k, v, ref_mask, int(S), int(W))
    compare(torch.from_numpy(out), ref, "C caller")
