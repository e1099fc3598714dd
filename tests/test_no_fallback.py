"""The product path has no CPU fallback and fails loudly (CPU-only checks).

* the binding refuses host tensors instead of computing anything on the CPU;
* a missing libdit.so is an error, not a silent switch to another path;
* without an sm_100 device every compute entry point of the C ABI returns
  DIT_ERR_UNSUPPORTED (this container has no GPU) once its arguments are valid;
* the binding never imports the oracle.
"""
import ctypes
import importlib
import sys

import pytest
import torch

import diffusion_transformer_denoising_dit_b200 as dit
from diffusion_transformer_denoising_dit_b200 import _binding as B

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="checks the behaviour on a host without a GPU")

DIT_ERR_UNSUPPORTED = 2
A16 = 1 << 20  # a fake 16-byte aligned device address (never dereferenced: the device check comes first)


def test_host_tensors_are_refused():
    q = torch.zeros(1, 1, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="no CPU path"):
        dit.attention(q, q, q)
    with pytest.raises(ValueError, match="no CPU path"):
        dit.fbcache_gate(torch.zeros(8, dtype=torch.bfloat16), torch.zeros(8, dtype=torch.bfloat16), 0.1)


def test_missing_library_is_an_error(monkeypatch):
    monkeypatch.setattr(B, "LIB_PATH", "/nonexistent/libdit.so")
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        B.lib()


def test_entry_points_report_unsupported_without_an_sm100_device():
    L = B.lib()
    st = B._i64x3(1024, 1024, 64)
    st8 = B._i64x3(16 * 128, 16 * 128, 128)
    O = A16 + (1 << 16)  # the output may not be an input
    args = (A16, A16, A16, O, 1, 1, 16, 64, st, st, st, st, None, None, 0.0)
    assert L.dit_attn_bf16(*args, None, 0, None) == DIT_ERR_UNSUPPORTED
    assert L.dit_attn_bf16_skippable(*args, None, 0, A16, None) == DIT_ERR_UNSUPPORTED
    args8 = (A16, A16, A16, O, 1, 1, 16, 128, st8, st8, st8, st8, None, None, 0.0)
    need = L.dit_attn_fp8_workspace_bytes(1, 1, 16, 128, 128, 64)
    assert L.dit_attn_fp8(*args8, 128, 64, 1, A16, need, None) == DIT_ERR_UNSUPPORTED
    assert L.dit_attn_fp8_i8qk(*args8, 128, 64, 1, A16, need, None) == DIT_ERR_UNSUPPORTED
    assert L.rope_apply(A16, A16, 1, 1, 16, 64, st, st, A16, A16, 0, None) == DIT_ERR_UNSUPPORTED
    assert L.dit_rope_tables(A16, 16, 16, 24, 24, 1e4, A16, A16, None) == DIT_ERR_UNSUPPORTED
    assert L.fbcache_gate(A16, A16, 64, 0.1, A16, A16, A16, 1 << 20, None) == DIT_ERR_UNSUPPORTED
    assert L.fbcache_gate_noalloc(A16, A16, 64, 0.1, A16, A16, None) == DIT_ERR_UNSUPPORTED
    assert L.fbcache_gate_sums(A16, A16, 64, A16, A16, 1 << 20, None) == DIT_ERR_UNSUPPORTED
    assert L.fbcache_gate_finalize(A16, 0.1, A16, A16, None) == DIT_ERR_UNSUPPORTED
    assert L.fbcache_gate_ref_update(A16, A16 + 4096, 64, None, None) == DIT_ERR_UNSUPPORTED
    assert L.dit_selftest_wait_timeout(None) == DIT_ERR_UNSUPPORTED
    assert L.dit_read_error(None) == DIT_ERR_UNSUPPORTED


def test_binding_does_not_import_the_oracle():
    for name in [m for m in sys.modules if m == "oracle" or m.startswith("oracle.")]:
        del sys.modules[name]
    importlib.reload(B)
    importlib.reload(dit)
    assert not any(m == "oracle" or m.startswith("oracle.") for m in sys.modules)


def test_binding_metadata_checks():
    """What the C ABI cannot see (table lengths, dtypes, devices) is checked before any call."""
    c = torch.zeros(10, 32)
    B._check_tables(None, None, 10, 64)
    B._check_tables(c, c, 10, 64)
    for bad in ((c, None), (c[:9], c[:9]), (c.double(), c.double()), (c.t().contiguous().t(), c)):
        with pytest.raises(ValueError):
            B._check_tables(*bad, 10, 64)
    with pytest.raises(ValueError):
        B._check_out(torch.zeros(1, 2, 10, 64), (1, 2, 10, 64), torch.bfloat16)
    with pytest.raises(ValueError):
        B._check_flags(torch.zeros(1, dtype=torch.float64), None)
    with pytest.raises(ValueError):
        B._check_flags(None, torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError):
        B._check_bytes(torch.zeros(4, 4, dtype=torch.uint8).t(), "workspace")
