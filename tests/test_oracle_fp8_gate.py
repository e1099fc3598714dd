"""Pins of the e4m3 quantiser and of the cache-gate oracle (no GPU)."""
import dataclasses
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


def test_block_quantisation_within_e4m3_error_bound():
    """Blocks six orders of magnitude apart, each with a planted amax: every scale is
    that amax / 448 exactly, and every dequantised element is within e4m3's rounding
    error of the input (half a step: 2^-4 |x| in the normal range, 2^-10 scale below
    it).  A scale taken from a neighbouring block saturates or underflows there."""
    x = rng.uniform(-1.0, 1.0, size=(1, 2, 300, 16))
    mags = np.array([1e3, 1e-3, 1e3, 1e-3, 1.0])
    amax = mags * 1.5
    for b in range(5):
        x[..., 64 * b:64 * (b + 1), :] *= mags[b]
        x[..., 64 * b + 7, 3] = -amax[b]
    codes, sc = fp8.quantize_blocks(x, 64)
    np.testing.assert_array_equal(sc, np.broadcast_to(amax / 448.0, sc.shape))
    rep = np.repeat(amax / 448.0, 64)[:300][None, None, :, None]
    err = np.abs(codes * rep - x)
    assert np.all(err <= 2.0 ** -4 * np.abs(x) + 2.0 ** -10 * rep)


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


# --------------------------------------------------------------------------- int8
# Symmetric per-block int8 for Q and K (SageAttention's 8-bit Q.K^T reading).
def test_int8_codes_round_trip_ties_to_even_and_clip():
    ints = np.arange(-127, 128, dtype=np.float64)
    np.testing.assert_array_equal(fp8.quantize_int8(ints), ints)
    mids = ints[:-1] + 0.5                                   # k + 1/2 for k = -127 .. 126
    lo = np.floor(mids)
    np.testing.assert_array_equal(fp8.quantize_int8(mids), np.where(lo % 2 == 0, lo, lo + 1))
    np.testing.assert_array_equal(fp8.quantize_int8([127.5, 1e9, -127.5, -1e9]), [127, 127, -127, -127])


def test_int8_matches_torch_round_and_clamp():
    x = rng.uniform(-140.0, 140.0, 50000)
    ref = torch.round(torch.from_numpy(x)).clamp(-127, 127).numpy()
    np.testing.assert_array_equal(fp8.quantize_int8(x), ref)


def test_int8_blocks_within_half_a_step():
    """Blocks six orders of magnitude apart with planted amax: scales exactly amax / 127,
    each block's amax on code +-127, every element within half a step (scale / 2), and
    an all-zero block gets scale 1."""
    x = rng.uniform(-1.0, 1.0, size=(1, 2, 300, 16))
    mags = np.array([1e3, 1e-3, 1e3, 1e-3, 1.0])
    amax = mags * 1.5
    for b in range(5):
        x[..., 64 * b:64 * (b + 1), :] *= mags[b]
        x[..., 64 * b + 9, 5] = amax[b]
    codes, sc = fp8.quantize_int8_blocks(x, 64)
    np.testing.assert_array_equal(sc, np.broadcast_to(amax / 127.0, sc.shape))
    rep = np.repeat(amax / 127.0, 64)[:300][None, None, :, None]
    assert np.all(np.abs(codes * rep - x) <= 0.5 * rep * (1 + 1e-12))
    for b in range(5):
        assert np.abs(codes[..., 64 * b:64 * (b + 1), :]).max() == 127.0
    assert fp8.quantize_int8_blocks(np.zeros((1, 1, 64, 4)), 64)[1][0, 0, 0] == 1.0


def _int8_exact_inputs(N=192, seed=21):
    """Inputs every step of the int8 reading represents exactly: integer Q, K with block
    amax 127 (scale 1), e4m3 V with block amax 448 (scale 1, no V fold), and scores
    k_j * ln 2 with k_j in [113, 127], so every P = 2^(k_j - 127) * 448 is an e4m3 value."""
    g = np.random.default_rng(seed)
    q = np.zeros((1, 1, N, 2))
    q[..., 0] = 127.0                                          # every query row the same
    k = np.zeros((1, 1, N, 2))
    k[..., 0] = g.integers(113, 128, N)
    k[..., 1] = g.integers(-127, 128, N)                       # meets q's zero channel
    k[..., ::64, 0] = 127.0                                    # block amax 127
    vals = _all_finite_values()
    v = g.choice(vals[np.abs(vals) <= 448.0], size=(1, 1, N, 2))
    v[..., ::64, 1] = 448.0                                    # block amax 448
    return q, k, v, math.log(2.0) / 127.0


def test_simulated_int8_is_exact_where_every_step_is():
    q, k, v, sigma = _int8_exact_inputs()
    exact = A.attention(q, k, v, scale=sigma)
    sim = fp8.simulated_attention(q, k, v, scale=sigma, smooth=False, qk="int8")
    np.testing.assert_allclose(sim, exact, rtol=1e-13, atol=1e-13)
    sim_e4m3 = fp8.simulated_attention(q, k, v, scale=sigma, smooth=False)
    assert np.abs(sim_e4m3 - exact).max() > 1e-3            # e4m3 Q.K^T is not exact here


def test_simulated_int8_keeps_an_integer_tie():
    """q = (127, 113) meets keys (127, 0) and (14, 127) with the same integer product
    16129; every other key is 0 (score 40 lower, its P rounds to 0) and V picks e0 / e1.
    The int8 reading, exact on these integers, gives (1/2, 1/2) on every row.  At scale
    127/448, 113 and 14 fall off the e4m3 grid by different relative amounts, so
    rounding Q, K or both to e4m3 breaks the tie."""
    N = 64
    q = np.zeros((1, 1, N, 2))
    q[...] = (127.0, 113.0)
    k = np.zeros((1, 1, N, 2))
    k[0, 0, 0] = (127.0, 0.0)
    k[0, 0, 1] = (14.0, 127.0)
    v = np.zeros((1, 1, N, 2))
    v[0, 0, 0] = (1.0, 0.0)
    v[0, 0, 1] = (0.0, 1.0)
    sigma = 40.0 / 16129.0
    o = fp8.simulated_attention(q, k, v, scale=sigma, smooth=False, qk="int8")
    np.testing.assert_allclose(o, 0.5, rtol=0, atol=1e-13)
    o8 = fp8.simulated_attention(q, k, v, scale=sigma, smooth=False)
    assert np.abs(o8 - 0.5).max() > 1e-2


def test_simulated_int8_meets_the_target_on_outliers():
    """Diagnostic (not a pin): on the 1024-px outlier workload the int8 Q.K^T reading
    reaches cosine >= 0.995 against exact attention, where e4m3 Q.K^T stays near 0.98."""
    w = synth.WORKLOADS["flux1k"]
    q, k, v = synth.qkv(dataclasses.replace(w, H=1))
    pos = synth.positions(w.T, w.G).numpy()
    rows = np.random.default_rng(4).integers(0, w.N, 128)
    ex = A.attention(q, k, v, pos=pos, axes=w.axes, theta=w.theta, rows=rows)
    cos = lambda a: float((a * ex).sum() / math.sqrt((a * a).sum() * (ex * ex).sum()))
    i8 = fp8.simulated_attention(q, k, v, pos=pos, axes=w.axes, theta=w.theta, rows=rows, qk="int8")
    e4 = fp8.simulated_attention(q, k, v, pos=pos, axes=w.axes, theta=w.theta, rows=rows)
    assert cos(i8) >= 0.995 > cos(e4)


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


# --- simulated_attention: closed forms and invariants of the FP8 reading -------------
# Each pin takes the implementation as an argument, so that the planted-mistake test
# below can run the same pins against mutated copies of the oracle.


def _dequant_rows(v, block=64):
    """V as the FP8 scheme sees it: e4m3 codes times their block scale."""
    codes, sc = fp8.quantize_blocks(v, block)
    return codes * np.repeat(sc, block, axis=-1)[..., : v.shape[-2], None]


def _pin_q_zero(sim):
    """Q = 0: every score is 0 and p = 1.  The second V block's scale is half the
    first's, so its P is 448 * 0.5 = 224, still exact in e4m3, and O is the plain
    mean of the dequantised V: P * v8 * sV_max / 448 = sV(j) * v8."""
    rng = np.random.default_rng(11)
    v = rng.uniform(-1.0, 1.0, size=(1, 1, 128, 16))
    v[0, 0, 3, 5] = 4.0       # block 0 amax 4
    v[0, 0, 70, 2] = -2.0     # block 1 amax 2: half the scale
    q = np.zeros_like(v)
    k = rng.standard_normal(v.shape)
    o = sim(q, k, v, smooth=False)
    want = _dequant_rows(v).mean(axis=-2, keepdims=True)
    np.testing.assert_allclose(o, np.broadcast_to(want, o.shape), rtol=0, atol=1e-14)


def _pin_one_hot(sim):
    """K = a I, Q rows = b e_pi(i) with sigma a b = 40: exp(-40) * 448 quantises to 0,
    so each output row is the dequantised V row of its partner key."""
    d, n = 64, 64
    a, b = 64.0, 40.0
    k = (a * np.eye(d))[None, None]
    perm = np.random.default_rng(12).permutation(n)
    q = (b * np.eye(d)[perm])[None, None]
    v = np.random.default_rng(13).standard_normal((1, 1, n, d))
    o = sim(q, k, v, scale=40.0 / (a * b), smooth=False)
    np.testing.assert_allclose(o, _dequant_rows(v)[:, :, perm], rtol=1e-14, atol=1e-14)


def _pin_block_permutation(sim):
    """Moving whole 64-key blocks of K and V together moves their scales with them."""
    rng = np.random.default_rng(14)
    q, k, v = (rng.standard_normal((1, 2, 256, 32)) for _ in range(3))
    k[..., 5] *= 8.0
    q[..., 5] *= 8.0
    idx = np.concatenate([np.arange(64 * b, 64 * (b + 1)) for b in (2, 0, 3, 1)])
    np.testing.assert_allclose(sim(q, k[:, :, idx], v[:, :, idx]), sim(q, k, v), rtol=1e-12, atol=1e-12)


def _pin_powers_of_two(sim):
    """V * 4 scales every V block scale by 4 with the same codes: O * 4 exactly; Q * 2
    with sigma / 2 leaves every score unchanged: the same O exactly."""
    rng = np.random.default_rng(15)
    q, k, v = (rng.standard_normal((1, 1, 192, 32)) for _ in range(3))
    o = sim(q, k, v, scale=0.2)
    assert np.array_equal(sim(q, k, 4.0 * v, scale=0.2), 4.0 * o)
    assert np.array_equal(sim(2.0 * q, k, v, scale=0.1), o)


def _pin_q_blocks(sim):
    """Scaling the rows of the second 128-token Q block by 4 scales only that block's
    Q scale (same codes): its rows equal those computed with 4 sigma, the first
    block's rows do not move."""
    rng = np.random.default_rng(16)
    q, k, v = (rng.standard_normal((1, 1, 256, 32)) for _ in range(3))
    q2 = q.copy()
    q2[:, :, 128:] *= 4.0
    o = sim(q, k, v, scale=0.1)
    o2 = sim(q2, k, v, scale=0.1)
    o4 = sim(q, k, v, scale=0.4)
    assert np.array_equal(o2[:, :, :128], o[:, :, :128])
    assert np.array_equal(o2[:, :, 128:], o4[:, :, 128:])


_SIM_PINS = [_pin_q_zero, _pin_one_hot, _pin_block_permutation, _pin_powers_of_two, _pin_q_blocks]


@pytest.mark.parametrize("pin", _SIM_PINS, ids=lambda f: f.__name__[5:])
def test_simulated_attention_pins(pin):
    pin(fp8.simulated_attention)


# plausible mistakes, planted in a copy of the oracle's own source (CPU only)
_SIM_MUTATIONS = {
    "per_head_v_max_replaced": ("* (svmax / E4M3_MAX) / l", "* (svc.mean() / E4M3_MAX) / l"),
    "row_sum_over_quantised_p": ("/ l\n", "/ (p8.sum(axis=1, keepdims=True) * 2.0)\n"),
    "kv_block_scale_misindexed": ("svc = np.repeat(sv[b, h], kv_block)[:N]",
                                  "svc = np.roll(np.repeat(sv[b, h], kv_block)[:N], 1)"),
    "q_block_scale_misindexed": ("sqr = np.repeat(sq[b, h], q_block)[:N]",
                                 "sqr = np.roll(np.repeat(sq[b, h], q_block)[:N], q_block)"),
    "sigma_dropped": ("s = sigma * (q8", "s = 1.0 * (q8"),
    "v_scale_not_folded_into_p": ("quantize_e4m3(p * (E4M3_MAX * svc / svmax)[None, :])",
                                  "quantize_e4m3(p * E4M3_MAX)"),
}


@pytest.mark.parametrize("name", sorted(_SIM_MUTATIONS))
def test_simulated_attention_pins_catch_planted_mistakes(name):
    import inspect
    old, new = _SIM_MUTATIONS[name]
    src = inspect.getsource(fp8.simulated_attention)
    assert old in src, name
    ns = dict(vars(fp8))
    exec(src.replace(old, new, 1), ns)
    mutant = ns["simulated_attention"]
    failed = 0
    for pin in _SIM_PINS:
        try:
            pin(mutant)
        except AssertionError:
            failed += 1
    assert failed >= 1, name


@pytest.mark.parametrize("pin", _SIM_PINS, ids=lambda f: f.__name__[5:])
def test_simulated_attention_int8_pins(pin):
    """The closed forms and invariants hold for the int8 Q.K^T reading too."""
    import functools
    pin(functools.partial(fp8.simulated_attention, qk="int8"))
