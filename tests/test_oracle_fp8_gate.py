"""Pins of the e4m3 quantiser and of the cache-gate oracle (no GPU)."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import fp8, gate
from oracle import attention as A
from diffusion_transformer_denoising_dit_b200 import synth

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")))
rng = np.random.default_rng(3)


# --------------------------------------------------------------------------- e4m3
def _all_finite_values():
    vals = [fp8.e4m3_decode(c) for c in range(256)]
    return np.array([v for v in vals if not math.isnan(v)])


def test_code_table_round_trip():
    vals = _all_finite_values()
    assert len(vals) == 254
    assert len(set(vals.tolist())) == 253          # +0 and -0
    assert vals.max() == 448.0 and vals.min() == -448.0
    np.testing.assert_array_equal(fp8.quantize_e4m3(vals), vals)


def test_ties_round_to_even_mantissa():
    pos = np.unique(_all_finite_values()[_all_finite_values() >= 0])
    mids = (pos[:-1] + pos[1:]) / 2
    got = fp8.quantize_e4m3(mids)
    for lo, hi, g in zip(pos[:-1], pos[1:], got):
        even = lo if (int(np.round(lo / _spacing(lo))) % 2 == 0) else hi
        assert g == even, (lo, hi, g)


def _spacing(x):
    e = max(math.floor(math.log2(x)) if x > 0 else -6, -6)
    return 2.0 ** (e - 3)


def test_golden_e4m3():
    for case in GOLD["e4m3"]:
        assert fp8.quantize_e4m3(case["x"]) == case["expect"], case


def test_matches_torch_float8_cast():
    x = np.concatenate([rng.standard_normal(20000) * s for s in (1e-3, 0.1, 3, 60, 400)])
    x = np.clip(x, -448, 448)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(fp8.quantize_e4m3(x), ref)


def test_saturation():
    np.testing.assert_array_equal(fp8.quantize_e4m3([1e9, -500.0, 449.0]), [448.0, -448.0, 448.0])


def test_block_scales_put_block_amax_on_448():
    x = rng.standard_normal((2, 3, 300, 64))
    q8, sc = fp8.quantize_blocks(x, 64)
    assert sc.shape == (2, 3, 5)
    for i in range(5):
        blk = q8[:, :, i * 64:(i + 1) * 64]
        np.testing.assert_array_equal(np.abs(blk).max(axis=(-2, -1)), 448.0)
    z = np.zeros((1, 1, 64, 8))
    assert fp8.block_scales(z, 64)[0, 0, 0] == 1.0


def test_smoothing_leaves_exact_attention_unchanged():
    q, k, v = (rng.standard_normal((1, 2, 80, 32)) for _ in range(3))
    k = k + 5.0
    np.testing.assert_allclose(A.attention(q, fp8.smooth_k(k), v), A.attention(q, k, v), atol=1e-12)


def test_simulated_fp8_is_close_to_exact():
    """Diagnostic sanity (not a parity pin): the quantisation floor is small on N(0,1) inputs."""
    q, k, v = (rng.standard_normal((1, 2, 256, 64)) for _ in range(3))
    o = A.attention(q, k, v)
    s = fp8.simulated_attention(q, k, v)
    cos = (o * s).sum() / np.sqrt((o * o).sum() * (s * s).sum())
    assert cos > 0.995


# --------------------------------------------------------------------------- gate
def test_golden_gate():
    for case in GOLD["gate"]:
        cur = torch.tensor(case["cur"], dtype=torch.bfloat16)
        prev = torch.tensor(case["prev"], dtype=torch.bfloat16)
        assert torch.equal(cur.double(), torch.tensor(case["cur"], dtype=torch.float64))  # bf16-exact
        assert gate.relative_l1(cur, prev) == case["rel"]


def test_gate_brute_force_on_tiny_sweep():
    for eps in (1e-4, 1e-2, 0.3):
        cur, prev = synth.gate_pair(288, 128, eps)
        r = gate.relative_l1(cur, prev)
        r2 = gate.relative_l1_loops(cur, prev)
        assert abs(r - r2) <= 1e-12 * max(r, 1e-30)


def test_gate_zero_denominator():
    z = np.zeros(10)
    assert gate.relative_l1(z, z) == 0.0 and gate.skip(0.0, 0.08)
    assert gate.relative_l1(np.ones(10), z) == math.inf and not gate.skip(math.inf, 0.08)


def test_gate_strict_threshold():
    assert gate.skip(0.0799999, 0.08)
    assert not gate.skip(0.08, 0.08)


def test_gate_symmetric_scaling():
    """rel is invariant to a common scale of both residuals (power-of-two scale keeps bf16 exact)."""
    cur, prev = synth.gate_pair(64, 32, 0.05)
    r = gate.relative_l1(cur, prev)
    assert gate.relative_l1(cur * 4, prev * 4) == r


def test_trace_decisions_follow_drift():
    res = list(synth.drift_residuals(96, 64, steps=28))
    dec = gate.trace_decisions(res, 0.12)
    assert dec[0][1] is False and len(dec) == 28
    sched = synth.drift_schedule(28)
    for k in range(1, 28):
        assert abs(dec[k][0] - sched[k - 1]) < 2e-3 * max(1.0, sched[k - 1] * 10)
    skipped = [k for k, (_, s) in enumerate(dec) if s]
    assert skipped == list(range(12, 28))


def _geometric_residuals(c, steps, shape=(16, 8), seed=0):
    """r_t = (1 + c)^t r_0 in fp64: against a reference k steps back, rel = (1 + c)^k - 1 exactly."""
    r0 = np.random.default_rng(seed).standard_normal(shape) + 3.0
    return [r0 * (1.0 + c) ** t for t in range(steps)]


def test_policy_consecutive_on_geometric_growth():
    """Each step changes by c = 0.05 < 0.12: every step after the warm-up is skipped."""
    res = _geometric_residuals(0.05, 12)
    dec = gate.trace_decisions(res, 0.12, policy="consecutive")
    assert [s for _, s in dec] == [False] + [True] * 11
    for _, (rel, _) in enumerate(dec[1:]):
        assert abs(rel - 0.05) < 1e-12


def test_policy_last_computed_accumulates_until_threshold():
    """Against the last computed step the change grows as (1.05)^k - 1: 0.05, 0.1025 (skip),
    0.157625 (compute), so exactly every third step runs."""
    res = _geometric_residuals(0.05, 13)
    dec = gate.trace_decisions(res, 0.12, policy="last_computed")
    computed = [t for t, (_, s) in enumerate(dec) if not s]
    assert computed == [0, 3, 6, 9, 12]
    assert abs(dec[3][0] - (1.05 ** 3 - 1.0)) < 1e-12
    assert abs(dec[4][0] - 0.05) < 1e-12  # the reference moved to step 3


def test_policy_warmup_forces_early_steps():
    res = _geometric_residuals(0.01, 8)
    dec = gate.trace_decisions(res, 0.12, warmup=5)
    assert [s for _, s in dec] == [False] * 5 + [True] * 3
    assert all(abs(rel - 0.01) < 1e-12 for rel, _ in dec[1:])


def test_policy_last_computed_on_the_drift_trace():
    """The decaying drift under the last-computed policy: changes accumulate across
    skipped steps, so fewer steps are skipped than with consecutive comparison, and
    every skipped step's accumulated change is below the threshold."""
    res = list(synth.drift_residuals(96, 64, steps=28))
    cons = gate.trace_decisions(res, 0.12)
    last = gate.trace_decisions(res, 0.12, policy="last_computed")
    n_cons = sum(s for _, s in cons)
    n_last = sum(s for _, s in last)
    assert 0 < n_last < n_cons
    ref = 0
    for t in range(1, 28):
        rel, s = last[t]
        assert abs(rel - gate.relative_l1(res[t], res[ref])) < 1e-15
        assert s == (rel < 0.12)
        if not s:
            ref = t


def test_policy_rejects_unknown_name():
    with pytest.raises(ValueError):
        gate.trace_decisions([np.ones(3)], 0.1, policy="nope")
