"""The debug build (libdit_debug.so, -DDIT_DEBUG): every kernel checks its
shared-memory, tensor-memory and TMA indices on the device and records
DIT_ERR_BOUNDS in the error word instead of making a bad access.  In place of a
sanitizer (closed on this pool), small and ragged cases of every entry point run
on it in a fresh process: no check may fire, and the results still match the
oracle.
"""
import os
import subprocess
import sys

import pytest

from conftest import ROOT, cuda_ok

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]

DEBUG_LIB = os.path.join(ROOT, "diffusion_transformer_denoising_dit_b200", "libdit_debug.so")

SCRIPT = r"""
import dataclasses, math, sys
import numpy as np, torch
import diffusion_transformer_denoising_dit_b200 as dit
from diffusion_transformer_denoising_dit_b200 import _binding, synth
from oracle import attention as A
from oracle import gate as G
assert _binding.LIB_PATH.endswith("libdit_debug.so"), _binding.LIB_PATH

def cos(a, b):
    return float((a * b).sum() / math.sqrt((a * a).sum() * (b * b).sum()))

def attn(w, N, prec, bar):
    q, k, v = synth.qkv(w, device="cuda", N=N, seed=N)
    Nn = q.shape[2]
    pos = synth.positions(w.T, int(math.isqrt(max(Nn - w.T, 1))) + 1)[:Nn]
    c, s = dit.rope_tables(pos.cuda(), w.axes, w.theta)
    o = dit.attention(q, k, v, c, s, precision=prec).cpu().double().numpy()
    assert dit.read_error() == 0, (w.name, N, prec)
    ref = A.attention(q.cpu(), k.cpu(), v.cpu(), pos=pos.numpy(), axes=w.axes, theta=w.theta)
    got = cos(o, ref)
    assert got >= bar, (w.name, N, prec, got)
    return got

tiny = synth.WORKLOADS["tiny"]
flux = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2, outliers=False)
for N in (1, 129, 288):
    attn(tiny, N, "bf16", 0.9999)
for N in (1, 129, 777):
    attn(flux, N, "bf16", 0.9999)
for prec in ("fp8", "fp8_i8qk"):
    for N in (1, 65, 700):
        attn(flux, N, prec, 0.995)
    # no rotary tables: the quantiser stages no table rows
    q, k, v = synth.qkv(flux, device="cuda", N=300, seed=300)
    o = dit.attention(q, k, v, None, None, precision=prec).cpu().double().numpy()
    assert dit.read_error() == 0, ("no rope", prec)
    assert cos(o, A.attention(q.cpu(), k.cpu(), v.cpu())) >= 0.995, ("no rope", prec)
cur, prev = synth.gate_pair(2049, 1, 1e-2, device="cuda")
rel, skip = dit.fbcache_gate(cur, prev, 0.05)
assert abs(rel.item() - G.relative_l1(cur.cpu(), prev.cpu())) <= 1e-6 * rel.item()
assert dit.read_error() == 0
print("debug build ok")
"""


@pytest.mark.skipif(not os.path.exists(DEBUG_LIB), reason="libdit_debug.so not built (run build())")
def test_debug_build_fires_no_bounds_check():
    env = dict(os.environ, DIT_LIB_VARIANT="debug", PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
    r = subprocess.run([sys.executable, "-c", SCRIPT], cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=600)
    assert r.returncode == 0 and "debug build ok" in r.stdout, (r.stdout[-2000:], r.stderr[-4000:])
