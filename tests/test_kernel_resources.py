"""Static resource checks of the sm_100a kernels (no GPU: nvcc cross-compiles).

* No kernel spills registers to local memory.
* The attention kernel's register re-split fits the registers the block is
  launched with: setmaxnreg.inc draws on threads x registers-per-thread at
  launch (what ptxas assigns), not on the SM's register file, and a split that
  asks for more waits forever.  The split's constants are read from the kernel
  source; the launch registers from ptxas.
"""
import os
import re
import shutil
import subprocess
import tempfile

import pytest

from diffusion_transformer_denoising_dit_b200 import build as BLD

pytestmark = pytest.mark.skipif(shutil.which("nvcc") is None and not os.path.exists("/usr/local/cuda/bin/nvcc"),
                                reason="nvcc not available")


def _ptxas_report(src: str) -> str:
    with tempfile.TemporaryDirectory() as tmp:
        cmd = [BLD._nvcc(), *BLD.ARCH, *BLD.FLAGS, "-Xptxas", "-v", "-c", os.path.join(BLD.CSRC, src),
               "-o", os.path.join(tmp, "k.o")]
        r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr
    return r.stdout + r.stderr


def _entries(report: str):
    """{mangled entry name: registers} from ptxas -v output."""
    out, cur = {}, None
    for line in report.splitlines():
        m = re.search(r"Compiling entry function '(\w+)'", line)
        if m:
            cur = m.group(1)
        m = re.search(r"Used (\d+) registers", line)
        if m and cur is not None:
            out[cur] = int(m.group(1))
            cur = None
    return out


@pytest.fixture(scope="module")
def reports():
    return {src: _ptxas_report(src) for src in BLD.SOURCES}


def test_every_source_compiles_its_kernels(reports):
    for src, rep in reports.items():
        if src == "capi.cu":
            continue
        assert _entries(rep), src


# Known spills, per kernel: (store bytes, load bytes) allowed.  None at present.
SPILL_ALLOWANCE: dict = {}


def test_no_register_spills(reports):
    for src, rep in reports.items():
        entry = None
        for line in rep.splitlines():
            m = re.search(r"Compiling entry function '(\w+)'", line)
            if m:
                entry = m.group(1)
            m = re.search(r"(\d+) bytes spill stores, (\d+) bytes spill loads", line)
            if not m:
                continue
            st, ld = int(m.group(1)), int(m.group(2))
            allow = next((v for k, v in SPILL_ALLOWANCE.items() if entry and k in entry), (0, 0))
            assert st <= allow[0] and ld <= allow[1], (src, entry, line.strip())


def test_register_resplit_fits_the_launch_registers(reports):
    text = open(os.path.join(BLD.CSRC, "attn_kernel.cuh")).read()
    threads = int(re.search(r"kThreads\s*=\s*(\d+)", text).group(1))
    soft = int(re.search(r"kRegsSoftmax\s*=\s*(\d+)", text).group(1))
    aux = int(re.search(r"kRegsAux\s*=\s*(\d+)", text).group(1))
    assert threads == 3 * 128                      # two softmax warpgroups + one producer/MMA warpgroup
    need = 2 * 128 * soft + 128 * aux
    found = 0
    for src in ("attn_bf16.cu", "attn_fp8.cu"):
        for name, regs in _entries(reports[src]).items():
            if "attn_kernel" not in name:
                continue
            found += 1
            assert need <= threads * regs, (name, regs, need, threads * regs)
    assert found == 4  # <bf16, 64>, <bf16, 128>, <fp8, 128>, <fp8, 128, integer Q.K^T>
