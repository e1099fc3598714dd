"""fbcache_gate_noalloc: the cache gate for callers that cannot hand the library
device memory (a plug-in whose host framework owns the device allocator, or a
step loop that must not allocate while it runs).  Its scratch is a fixed array
inside the library instead of a workspace argument.

Checked through the C ABI against fbcache_gate on the same inputs, on two calls
in a row (the second call must not see anything left over from the first).
This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from conftest import cuda_ok
from diffusion_transformer_denoising_dit_b200 import _binding, synth

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


def _with_workspace(L, cur, prev, thr):
    n = cur.numel()
    ws = torch.empty(L.fbcache_gate_workspace_bytes(n), dtype=torch.uint8, device="cuda")
    rel = torch.empty(1, dtype=torch.float32, device="cuda")
    skip = torch.empty(1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert L.fbcache_gate(cur.data_ptr(), prev.data_ptr(), n, thr, rel.data_ptr(), skip.data_ptr(),
                          ws.data_ptr(), ws.numel(), st) == 0
    return rel, skip


def _no_alloc(L, cur, prev, thr):
    rel = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    skip = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert L.fbcache_gate_noalloc(cur.data_ptr(), prev.data_ptr(), cur.numel(), thr, rel.data_ptr(),
                                  skip.data_ptr(), st) == 0
    return rel, skip


def test_no_alloc_gate_matches_workspace_gate_twice():
    """Large n, then small n, then larger n again on the same stream: the small call
    leaves stale partials only in the slots the large calls overwrite, and the last
    call (every pass-1 slot up to the cap) must not read anything the small call
    left behind."""
    L = _binding.lib()
    cases = [(synth.gate_pair(4608, 3072, 0.3, seed=11, device="cuda"), 0.08),   # large change: compute
             (synth.gate_pair(288, 128, 1e-2, seed=12, device="cuda"), 0.08),    # small change, fewer CTAs: skip
             (synth.gate_pair(16896, 3072, 0.05, seed=13, device="cuda"), 0.12)]  # the benchmark's size, after it
    for (cur, prev), thr in cases:
        ref_rel, ref_skip = _with_workspace(L, cur, prev, thr)
        rel, skip = _no_alloc(L, cur, prev, thr)
        torch.cuda.synchronize()
        r, rr = rel.item(), ref_rel.item()
        assert abs(r - rr) <= 1e-6 * abs(rr)
        assert skip.item() == ref_skip.item()
    assert _binding.read_error() == 0


@pytest.mark.parametrize("n", [2047, 2048, 2049, 2056, 4097])
def test_no_alloc_gate_around_one_cta(n):
    """Sizes at and just past one pass-1 CTA's 2048 elements (one, then two CTAs)."""
    L = _binding.lib()
    cur, prev = synth.gate_pair(n, 1, 1e-2, seed=n, device="cuda")
    ref_rel, ref_skip = _with_workspace(L, cur, prev, 0.05)
    rel, skip = _no_alloc(L, cur, prev, 0.05)
    torch.cuda.synchronize()
    assert abs(rel.item() - ref_rel.item()) <= 1e-6 * abs(ref_rel.item())
    assert skip.item() == ref_skip.item()


def test_no_alloc_gate_rejects_bad_arguments():
    L = _binding.lib()
    x = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(2, dtype=torch.float32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert L.fbcache_gate_noalloc(x.data_ptr(), x.data_ptr(), 0, 0.1, out.data_ptr(), out.data_ptr(), st) == 1
    assert L.fbcache_gate_noalloc(x.data_ptr() + 2, x.data_ptr(), 8, 0.1, out.data_ptr(), out.data_ptr(), st) == 3
    # the same verdict as fbcache_gate on non-finite and extreme thresholds
    ws = torch.empty(L.fbcache_gate_workspace_bytes(64), dtype=torch.uint8, device="cuda")
    flt_max = torch.finfo(torch.float32).max
    for thr in (float("nan"), float("inf"), -float("inf"), flt_max, -flt_max):
        a = L.fbcache_gate(x.data_ptr(), x.data_ptr(), 64, thr, out.data_ptr(), out.data_ptr() + 4,
                           ws.data_ptr(), ws.numel(), st)
        b = L.fbcache_gate_noalloc(x.data_ptr(), x.data_ptr(), 64, thr, out.data_ptr(), out.data_ptr() + 4, st)
        assert a == b, (thr, a, b)
    torch.cuda.synchronize()
