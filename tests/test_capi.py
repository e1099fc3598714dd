"""C-ABI checks that need no GPU: the library loads, exports every symbol that
include/dit.h declares, and rejects bad arguments before touching a device."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

from diffusion_transformer_denoising_dit_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "dit.h")

pytestmark = pytest.mark.skipif(not os.path.exists(B.LIB_PATH), reason="libdit.so not built (run build())")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"DIT_API\s+[\w\s\*]+?\b(\w+)\s*\(", txt)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(B.EXPORTS)


def test_debug_build_exports_every_declared_symbol():
    path = os.path.join(os.path.dirname(B.LIB_PATH), "libdit_debug.so")
    if not os.path.exists(path):
        pytest.skip("libdit_debug.so not built (run build())")
    L = ctypes.CDLL(path)
    for name in _declared():
        assert hasattr(L, name), name


def test_library_exports_every_declared_symbol():
    L = B.lib()
    for name in _declared():
        assert hasattr(L, name), name


def test_status_strings():
    L = B.lib()
    for code, name in B.STATUS.items():
        assert L.dit_status_string(code).decode() == name


S = B._i64x3
A16 = 1 << 20          # a fake 16-byte aligned device address (never dereferenced)


def _attn(L, q=A16, k=A16, v=A16, o=A16 + 4096, Bn=1, H=1, N=16, d=64, s=(1024, 1024, 64), cos=None, sin=None,
          scale=0.0, ws=None, wsb=0):
    st = S(*s)
    return L.dit_attn_bf16(q, k, v, o, Bn, H, N, d, st, st, st, st, cos, sin, scale, ws, wsb, None)


def test_attention_argument_validation():
    L = B.lib()
    assert _attn(L, q=None) == 1                      # null pointer
    assert _attn(L, N=0) == 1                         # empty sequence
    assert _attn(L, d=96) == 2                        # unsupported head dim
    assert _attn(L, q=A16 + 2) == 3                   # misaligned base
    assert _attn(L, s=(1024, 1024, 60)) == 3          # token stride not 16-byte aligned
    assert _attn(L, cos=A16) == 3                     # only one of the two tables
    assert _attn(L, cos=A16, sin=A16) == 4            # RoPE needs a workspace
    need = L.dit_attn_bf16_workspace_bytes(1, 1, 16, 64, 1)
    assert need == 2 * 16 * 64                       # rotated K, bf16, 256-byte aligned (Q rotates in-kernel)
    assert _attn(L, cos=A16, sin=A16, ws=A16, wsb=need - 1) == 4
    assert L.dit_attn_bf16_workspace_bytes(1, 1, 16, 64, 0) == 0


def test_layout_validation_rejects_broadcast_and_overlap():
    """A dimension of extent > 1 must advance and token rows may not overlap; a
    zero stride on an extent-1 dimension is harmless."""
    L = B.lib()
    assert _attn(L, H=2, s=(1 << 20, 0, 64)) == 1       # heads broadcast
    assert _attn(L, Bn=2, s=(0, 1024, 64)) == 1         # batch broadcast
    assert _attn(L, s=(1024, 1024, 0)) == 1             # every token the same row
    assert _attn(L, s=(1024, 1024, 32)) == 1            # rows overlap (token stride < d)
    # legal layouts get past the layout check to the workspace check (no device call)
    assert _attn(L, s=(0, 0, 64), cos=A16, sin=A16) == 4                   # B = H = 1
    assert _attn(L, H=4, s=(16 * 4 * 64, 64, 4 * 64), cos=A16, sin=A16) == 4  # [B, N, H, d]


def test_output_may_not_be_an_input():
    L = B.lib()
    for name in ("q", "k", "v"):
        assert _attn(L, **{name: A16 + 4096}, o=A16 + 4096) == 1
    st = S(1 << 20, 1 << 20, 128)
    args = (A16, A16, A16, A16, 1, 1, 1024, 128, st, st, st, st, None, None, 0.0, 128, 64, 1, A16, 1 << 30, None)
    assert L.dit_attn_fp8(*args) == 1                    # o == q


def test_rope_apply_in_place_needs_equal_strides():
    L = B.lib()
    a, b = S(4096, 4096, 64), S(8192, 4096, 64)
    assert L.rope_apply(A16, A16, 2, 1, 64, 64, a, b, A16, A16, 0, None) == 1


def test_small_outputs_alignment():
    L = B.lib()
    assert L.fbcache_gate(A16, A16, 100, 0.1, A16 + 2, A16, A16, 1 << 20, None) == 3    # rel_out
    assert L.fbcache_gate(A16, A16, 100, 0.1, A16, A16 + 1, A16, 1 << 20, None) == 3    # skip_out
    assert L.fbcache_gate_noalloc(A16, A16, 100, 0.1, A16 + 2, A16, None) == 3
    assert L.fbcache_gate_finalize(A16, 0.1, A16, A16 + 2, None) == 3
    assert L.dit_rope_tables(A16 + 2, 10, 16, 24, 24, 1e4, A16, A16, None) == 3        # pos


def test_gate_reference_update_argument_checks():
    L = B.lib()
    assert L.fbcache_gate_ref_update(None, A16, 64, None, None) == 1          # null input
    assert L.fbcache_gate_ref_update(A16, A16, 64, None, None) == 1           # r_ref == r_cur
    assert L.fbcache_gate_ref_update(A16, A16 + 4096, 0, None, None) == 1     # n < 1
    assert L.fbcache_gate_ref_update(A16 + 2, A16 + 4096, 64, None, None) == 3
    assert L.fbcache_gate_ref_update(A16, A16 + 4096, 64, A16 + 2, None) == 3  # misaligned flag


def test_integer_qk_variant_shares_the_fp8_argument_checks():
    L = B.lib()
    st = S(1 << 20, 1 << 20, 128)
    args = (A16, A16, A16, A16 + (1 << 24), 1, 1, 1024, 128, st, st, st, st, None, None, 0.0)
    assert L.dit_attn_fp8_i8qk(*args, 64, 64, 1, A16, 1 << 30, None) == 2     # q_block != 128
    assert L.dit_attn_fp8_i8qk(*args, 128, 64, 1, None, 0, None) == 4         # no workspace
    args64 = (A16, A16, A16, A16 + (1 << 24), 1, 1, 1024, 64, st, st, st, st, None, None, 0.0)
    assert L.dit_attn_fp8_i8qk(*args64, 128, 64, 1, A16, 1 << 30, None) == 2  # d = 64


def test_gate_entry_points_agree_on_thresholds():
    """fbcache_gate and fbcache_gate_noalloc accept and refuse the same thresholds:
    NaN and +-inf are refused, every finite float (FLT_MAX included) passes the
    argument checks (and then meets the device check, with no GPU here)."""
    L = B.lib()
    flt_max = float(np.finfo(np.float32).max)
    for thr in (float("nan"), float("inf"), -float("inf"), flt_max, -flt_max, 3.4e38, 0.0, 0.12):
        a = L.fbcache_gate(A16, A16, 100, thr, A16, A16, A16, 1 << 20, None)
        b = L.fbcache_gate_noalloc(A16, A16, 100, thr, A16, A16, None)
        assert a == b, (thr, a, b)
        assert a == (1 if not math.isfinite(thr) else 2), (thr, a)


def test_skippable_attention_argument_validation():
    L = B.lib()
    st = S(1024, 1024, 64)
    args = (A16, A16, A16, A16, 1, 1, 16, 64, st, st, st, st, None, None, 0.0, None, 0)
    assert L.dit_attn_bf16_skippable(*args, None, None) == 1      # the flag is required
    assert L.dit_attn_bf16_skippable(*args, A16 + 2, None) == 3   # 4-byte aligned flag


def test_fp8_argument_validation():
    L = B.lib()
    st = S(1024 * 128, 1024 * 128, 128)
    args = (A16, A16, A16, A16 + 4096, 1, 1, 1024, 128, st, st, st, st, None, None, 0.0)
    assert L.dit_attn_fp8(*args, 64, 64, 1, A16, 1 << 30, None) == 2      # q_block != 128
    assert L.dit_attn_fp8(*args, 128, 64, 1, None, 0, None) == 4          # no workspace
    small = L.dit_attn_fp8_workspace_bytes(1, 1, 1024, 128, 128, 64) - 1
    assert L.dit_attn_fp8(*args, 128, 64, 1, A16, small, None) == 4
    big = S(40000 * 1024 * 128, 1024 * 128, 128)
    wide = (A16, A16, A16, A16 + 4096, 2, 40000, 1024, 128, big, big, big, big, None, None, 0.0)
    assert L.dit_attn_fp8(*wide, 128, 64, 1, None, 0, None) == 2          # B * H > 65535 (before the workspace)


def test_gate_and_rope_validation():
    L = B.lib()
    assert L.fbcache_gate(A16, A16, 0, 0.1, A16, A16, A16, 1 << 20, None) == 1      # n = 0
    assert L.fbcache_gate(A16 + 4, A16, 100, 0.1, A16, A16, A16, 1 << 20, None) == 3
    assert L.fbcache_gate(A16, A16, 100, 0.1, A16, A16, A16, 1, None) == 4           # workspace too small
    assert L.fbcache_gate_workspace_bytes(100) == 16
    assert L.dit_rope_tables(A16, 10, 16, 24, 25, 1e4, A16, A16, None) == 1          # odd axis width
    assert L.dit_rope_tables(A16, 10, 16, 24, 24, -1.0, A16, A16, None) == 1         # bad theta
    st = S(4096, 4096, 64)
    assert L.rope_apply(A16, A16, 1, 1, 64, 64, st, st, A16, A16, 1, None) == 1      # fp32 out in place
    assert L.rope_apply(A16, A16, 1, 1, 64, 48, st, st, A16, A16, 0, None) == 2      # d = 48


def test_no_gpu_means_unsupported_not_fallback():
    torch = pytest.importorskip("torch")
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    L = B.lib()
    assert _attn(L) == 2
    assert L.fbcache_gate(A16, A16, 100, 0.1, A16, A16, A16, 1 << 20, None) == 2


def test_unit_rate_probe_argument_checks():
    """dit_probe_unit_rates refuses a null output or too small a capacity before
    touching a device; without a GPU it reports unsupported."""
    L = B.lib()
    buf = (ctypes.c_double * 4)()
    assert L.dit_probe_unit_rates(None, 4, None) == 1
    assert L.dit_probe_unit_rates(ctypes.cast(buf, ctypes.c_void_p), 3, None) == 1
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        assert L.dit_probe_unit_rates(ctypes.cast(buf, ctypes.c_void_p), 4, None) == 2
