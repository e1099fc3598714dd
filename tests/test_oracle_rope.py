"""Pins of the fp64 rotary-embedding oracle (no GPU).

Definition pinned: multi-axis rotary embedding with interleaved channel pairs
([vflash] "Optimization ledger", row "strict Triton RoPE"; see oracle/rope.py).
"""
import json
import os

import numpy as np
import pytest

from oracle import rope
from diffusion_transformer_denoising_dit_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))
rng = np.random.default_rng(11)
AX128 = (16, 56, 56)
AX64 = (16, 24, 24)


def test_golden_hand_values():
    for case in GOLD["rope"]:
        d = sum(case["axes"])
        x = np.zeros((1, d))
        p = case["pair"]
        x[0, 2 * p:2 * p + 2] = case["x"]
        y = rope.apply(x, np.array([case["pos"]]), case["axes"], case["theta"])
        np.testing.assert_allclose(y[0, 2 * p:2 * p + 2], case["expect"], rtol=0, atol=1e-15)
        others = np.delete(y[0], [2 * p, 2 * p + 1])
        assert np.all(others == 0)


def test_matches_complex_multiplication():
    """Independent formulation: pair (x0, x1) as x0 + i x1 times exp(i * pos_a * theta^(-2p/d_a))."""
    pos = synth.positions(5, 6).numpy()
    x = rng.standard_normal((3, pos.shape[0], 128))
    y = rope.apply(x, pos, AX128)
    z = x[..., 0::2] + 1j * x[..., 1::2]
    off = 0
    for a, da in enumerate(AX128):
        for p in range(da // 2):
            w = np.exp(1j * pos[:, a] * (10000.0 ** (-(2 * p) / da)))
            z[..., off // 2 + p] *= w
        off += da
    np.testing.assert_allclose(y[..., 0::2], z.real, atol=1e-13)
    np.testing.assert_allclose(y[..., 1::2], z.imag, atol=1e-13)


def test_pair_norms_preserved():
    pos = synth.positions(32, 16).numpy()
    x = rng.standard_normal((2, pos.shape[0], 64))
    y = rope.apply(x, pos, AX64)
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-13)


def test_position_zero_is_identity():
    x = rng.standard_normal((4, 10, 128))
    np.testing.assert_array_equal(rope.apply(x, np.zeros((10, 3), int), AX128), x)


def test_inverse_rotation():
    pos = synth.positions(16, 8).numpy()
    x = rng.standard_normal((pos.shape[0], 64))
    y = rope.apply(x, pos, AX64)
    back = rope.apply(y, -pos, AX64)
    np.testing.assert_allclose(back, x, atol=1e-12)


@pytest.mark.parametrize("shift", [(3, 0, 0), (0, 5, 0), (0, 0, 7), (2, 9, 4)])
def test_scores_depend_only_on_relative_position(shift):
    pos = rng.integers(0, 60, size=(40, 3))
    q = rng.standard_normal((40, 128))
    k = rng.standard_normal((40, 128))
    s0 = rope.apply(q, pos, AX128) @ rope.apply(k, pos, AX128).T
    pos2 = pos + np.array(shift)
    s1 = rope.apply(q, pos2, AX128) @ rope.apply(k, pos2, AX128).T
    np.testing.assert_allclose(s1, s0, atol=1e-11)


def test_axes_are_independent():
    """Moving only the axis-1 position leaves channels outside axis 1 untouched."""
    x = rng.standard_normal((1, 128))
    a = rope.apply(x, np.array([[4, 0, 2]]), AX128)
    b = rope.apply(x, np.array([[4, 9, 2]]), AX128)
    np.testing.assert_array_equal(a[:, :16], b[:, :16])
    np.testing.assert_array_equal(a[:, 72:], b[:, 72:])
    assert not np.allclose(a[:, 16:72], b[:, 16:72])


def test_angles_table_layout():
    ang = rope.angles(np.array([[2, 3, 5]]), AX64)
    assert ang.shape == (1, 32)
    np.testing.assert_allclose(ang[0, 0], 2.0)          # axis 0, pair 0
    np.testing.assert_allclose(ang[0, 8], 3.0)          # axis 1, pair 0 (offset 16 -> pair 8)
    np.testing.assert_allclose(ang[0, 20], 5.0)         # axis 2, pair 0 (offset 40 -> pair 20)
    np.testing.assert_allclose(ang[0, 9], 3.0 * 10000.0 ** (-2 / 24))
