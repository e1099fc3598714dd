"""NVTX ranges of the C ABI, checked without a GPU.

Every entry point that launches work (and dit_read_error) opens one NVTX range
named after itself and closes it on return.  A small NVTX tool
(tests/nvtx_probe.c, built here with gcc) is loaded by the NVTX loader inside
libdit.so through NVTX_INJECTION64_PATH and records every push and pop.  Calls
with arguments the library rejects return before touching a device, so the
ranges can be observed on a host without a GPU.
"""
import os
import shutil
import subprocess
import sys

import pytest

from diffusion_transformer_denoising_dit_b200 import _binding as B

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CUDA_INCLUDE = "/usr/local/cuda/include"

pytestmark = [
    pytest.mark.skipif(not os.path.exists(B.LIB_PATH), reason="libdit.so not built (run build())"),
    pytest.mark.skipif(shutil.which("gcc") is None or not os.path.exists(os.path.join(CUDA_INCLUDE, "nvtx3")),
                       reason="needs gcc and the NVTX v3 headers"),
]

SCRIPT = r"""
import ctypes, sys
from diffusion_transformer_denoising_dit_b200 import _binding as B
L = B.lib()
A16 = 1 << 20
st = B._i64x3(1024 * 128, 1024 * 128, 128)
args = (A16, A16, A16, A16 + 4096, 1, 1, 1024, 128, st, st, st, st, None, None, 0.0)
codes = [
    L.dit_attn_fp8(*args, 64, 64, 1, A16, 1 << 30, None),               # q_block != 128
    L.dit_attn_fp8_i8qk(*args, 64, 64, 1, A16, 1 << 30, None),
    L.dit_attn_bf16(A16, A16, A16, A16, 1, 1, 16, 64, st, st, st, st, None, None, 0.0, None, 0, None),  # o == q
    L.rope_apply(A16, A16, 2, 1, 64, 64, st, st, A16, A16, 7, None),     # dtype 7
    L.fbcache_gate(A16, A16, 0, 0.1, A16, A16, A16, 1 << 20, None),     # n = 0
]
probe = ctypes.CDLL(sys.argv[1])
probe.nvtx_probe_log.restype = ctypes.c_char_p
print(" ".join(str(c) for c in codes))
print(probe.nvtx_probe_log().decode(), end="")
"""


def test_each_call_is_one_named_nvtx_range(tmp_path):
    so = str(tmp_path / "libnvtx_probe.so")
    subprocess.run(["gcc", "-shared", "-fPIC", "-O1", "-I", CUDA_INCLUDE, os.path.join(HERE, "nvtx_probe.c"),
                    "-o", so], check=True, capture_output=True, text=True, timeout=120)
    env = dict(os.environ, NVTX_INJECTION64_PATH=so, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", SCRIPT, so], env=env, capture_output=True, text=True, timeout=300,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    lines = r.stdout.splitlines()
    codes = [int(c) for c in lines[0].split()]
    assert all(c != 0 for c in codes), codes   # every call was rejected on its arguments
    names = ["dit_attn_fp8", "dit_attn_fp8_i8qk", "dit_attn_bf16", "rope_apply", "fbcache_gate"]
    assert lines[1:] == [x for n in names for x in (n, "pop")], lines


def test_without_a_tool_the_calls_behave_the_same():
    env = {k: v for k, v in os.environ.items() if k != "NVTX_INJECTION64_PATH"}
    env["PYTHONPATH"] = ROOT + os.pathsep + os.environ.get("PYTHONPATH", "")
    script = SCRIPT.split("probe = ctypes.CDLL")[0] + "print(' '.join(str(c) for c in codes))\n"
    r = subprocess.run([sys.executable, "-c", script], env=env, capture_output=True, text=True, timeout=300,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr
    assert all(int(c) != 0 for c in r.stdout.split()), r.stdout
