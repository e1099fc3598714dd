"""Pins of the fp64 attention oracle against closed forms, invariants, brute force
and an independent library special case (no GPU).

Definition pinned: scaled dot-product attention over the joint token sequence
([VisualGen] "why the differences arise"; see oracle/attention.py).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import attention as A
from diffusion_transformer_denoising_dit_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))
rng = np.random.default_rng(7)


def _rand(B=1, H=2, N=40, d=16, scale=1.0):
    return [rng.standard_normal((B, H, N, d)) * scale for _ in range(3)]


def test_golden_hand_example():
    for case in GOLD["attention"]:
        q = np.array(case["q"])[None, None]
        k = np.array(case["k"])[None, None]
        v = np.array(case["v"])[None, None]
        o = A.attention(q, k, v)[0, 0]
        np.testing.assert_allclose(o, np.array(case["expect"]), rtol=0, atol=1e-14)


def test_zero_q_gives_mean_v_with_and_without_rope():
    q, k, v = _rand(N=50, d=64)
    q[:] = 0
    o = A.attention(q, k, v)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-13)
    pos = synth.positions(2, 7).numpy()[:50 - 1]
    pos = np.concatenate([pos, [[0, 9, 9]]])
    o2 = A.attention(q, k, v, pos=pos, axes=(16, 24, 24))
    np.testing.assert_allclose(o2, o, atol=1e-13)


def test_one_hot_scores_select_rows():
    N = d = 32
    c = 12.0        # sigma * c^2 = 144/sqrt(32) ~ 25.5 > 20 -> off-diagonal weight < e^-25
    basis = np.linalg.qr(rng.standard_normal((d, d)))[0]
    k = (c * basis)[None, None]
    perm = rng.permutation(N)
    q = k[:, :, perm, :]
    v = rng.standard_normal((1, 1, N, d))
    o = A.attention(q, k, v)
    np.testing.assert_allclose(o[0, 0], v[0, 0, perm], atol=1e-9)


def test_permutation_equivariance():
    q, k, v = _rand(N=37, d=16)
    p = rng.permutation(37)
    o = A.attention(q, k, v)
    o_kv = A.attention(q, k[:, :, p], v[:, :, p])
    np.testing.assert_allclose(o_kv, o, atol=1e-13)
    o_q = A.attention(q[:, :, p], k, v)
    np.testing.assert_allclose(o_q, o[:, :, p], atol=1e-13)


def test_single_token_returns_v():
    q, k, v = _rand(N=1, d=64)
    np.testing.assert_allclose(A.attention(q, k, v), v, atol=0)


def test_constant_v_gives_constant_output():
    q, k, v = _rand(N=33, d=16)
    v[:] = 1.75
    np.testing.assert_allclose(A.attention(q, k, v), 1.75, atol=1e-14)


def test_key_shift_invariance():
    q, k, v = _rand(N=45, d=32)
    m = rng.standard_normal((1, 2, 1, 32)) * 3
    np.testing.assert_allclose(A.attention(q, k + m, v), A.attention(q, k, v), atol=1e-12)


def test_matches_torch_sdpa_float64():
    q, k, v = _rand(B=2, H=3, N=70, d=64)
    o = A.attention(q, k, v, scale=0.3)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v), scale=0.3).numpy()
    np.testing.assert_allclose(o, ref, atol=1e-12)
    o_def = A.attention(q, k, v)
    ref_def = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    np.testing.assert_allclose(o_def, ref_def, atol=1e-12)


def test_brute_force_loops():
    q, k, v = _rand(B=1, H=1, N=6, d=4)
    np.testing.assert_allclose(A.attention(q, k, v), A.attention_loops(q, k, v), atol=1e-13)


def test_row_subset_matches_full():
    q, k, v = _rand(N=90, d=16)
    rows = np.array([0, 5, 89, 44])
    np.testing.assert_allclose(A.attention(q, k, v, rows=rows, chunk=3),
                               A.attention(q, k, v)[:, :, rows], atol=1e-14)


def test_rope_is_applied_to_q_and_k_not_v():
    """With RoPE, scores equal those of explicitly rotated Q, K; V passes through."""
    w = synth.WORKLOADS["tiny"]
    pos = synth.positions(w.T, w.G).numpy()
    q, k, v = (rng.standard_normal((1, 1, w.N, 64)) for _ in range(3))
    from oracle import rope
    qr = rope.apply(q, pos, w.axes)
    kr = rope.apply(k, pos, w.axes)
    np.testing.assert_allclose(A.attention(q, k, v, pos=pos, axes=w.axes),
                               A.attention(qr, kr, v), atol=1e-13)


def test_round_bf16_matches_torch_cast_of_float32():
    """fp32 -> bf16 in torch is a single round-to-nearest-even: an independent check."""
    x = np.concatenate([rng.standard_normal(50000) * s for s in (1e-3, 1.0, 37.0, 1e4)]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(A.round_bf16(x.astype(np.float64)), ref)


def test_round_bf16_ties_and_exact_values():
    # 1 + 2^-8 is half-way between 1 and 1 + 2^-7: ties to even (1.0)
    assert A.round_bf16(1.0 + 2.0 ** -8) == 1.0
    assert A.round_bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2 * 2.0 ** -7
    assert A.round_bf16(-3.0) == -3.0 and A.round_bf16(0.0) == 0.0


def test_bf16_operand_reading_is_rounded_rotation():
    w = synth.WORKLOADS["tiny"]
    pos = synth.positions(w.T, w.G).numpy()
    q, k, v = (rng.standard_normal((1, 1, w.N, 64)) for _ in range(3))
    from oracle import rope
    qr = A.round_bf16(rope.apply(q, pos, w.axes))
    kr = A.round_bf16(rope.apply(k, pos, w.axes))
    np.testing.assert_allclose(A.attention(q, k, v, pos=pos, axes=w.axes, operands="bf16"),
                               A.attention(qr, kr, v), atol=1e-14)


@pytest.mark.parametrize("mutation", ["no_scale", "transpose_v", "no_max_sub_row", "sum_over_queries"])
def test_pins_catch_planted_mistakes(mutation):
    """Plant plausible mistakes in a copy of the oracle's formula and check a pin fails."""
    def bad(q, k, v):
        s = q[0, 0] @ k[0, 0].T
        if mutation != "no_scale":
            s = s / math.sqrt(q.shape[-1])
        if mutation == "no_max_sub_row":
            s = s - s.max()          # harmless globally -> must still pass torch check
        else:
            s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        vv = v[0, 0].T if mutation == "transpose_v" else v[0, 0]
        z = e.sum(axis=0, keepdims=True).T if mutation == "sum_over_queries" else e.sum(axis=1, keepdims=True)
        return ((e @ vv) / z)[None, None]
    q, k, v = _rand(B=1, H=1, N=16, d=16)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()
    ok = np.allclose(bad(q, k, v), ref, atol=1e-10)
    if mutation == "no_max_sub_row":
        assert ok          # subtracting any constant is exact; the pin must not over-reject
    else:
        assert not ok
