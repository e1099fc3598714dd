"""A float32 model of the FP8 attention kernel's arithmetic, against the oracle (no GPU).

The model follows the kernel's softmax step by step, in fp32 where the kernel
computes in fp32, on the oracle's e4m3 codes and block scales:

* scores per 128-key tile: S = Q8 K8^T (exact e4m3 products, fp32 sum), scaled per
  64-key half by sQ * sK(half) * scale * log2(e);
* lazy rescale per warp of 32 rows: the running max moves only when some row's
  tile max exceeds it by more than tau = 4 (log2 units);
* P = 2^(x + log2 f - m) with f = sV(half) * 448 / (sV_max * 2^4), rounded to e4m3
  (RNE, saturating) -- the V block scale folded into the exponent;
* row sum of the unrounded P, each half divided by its f; O rescaled by
  2^(m_old - m_new) when the max moved; O += P8 V8; output O * sV_max * 2^4 / 448 / l.

It is the reference for the kernel's own arithmetic: it separates what the
scheme does (the simulated-FP8 oracle, exact row max, no headroom) from what the
kernel's stale max frame and headroom add, and a kernel output that differs from
it by more than rounding points at the kernel rather than at the scheme.
"""
import dataclasses
import math

import numpy as np

from oracle import attention as A
from oracle import fp8 as F
from oracle import rope as R
from diffusion_transformer_denoising_dit_b200 import synth

from fp8_kernel_arith import kernel_model  # noqa: E402


def _cos(a, b):
    return float((a * b).sum() / math.sqrt((a * a).sum() * (b * b).sum()))


def _case(outliers, qk="e4m3"):
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2, outliers=outliers)
    q, k, v = synth.qkv(w)
    pos = synth.positions(w.T, w.G).numpy()
    rows = np.unique(np.concatenate([np.arange(0, 128), np.random.default_rng(4).integers(0, w.N, 128)]))
    args = dict(pos=pos, axes=w.axes, theta=w.theta, rows=rows)
    exact = A.attention(q, k, v, **args)
    sim = F.simulated_attention(q, k, v, qk=qk, **args)
    model = kernel_model(q, k, v, pos, w.axes, w.theta, rows, qk=qk)
    return exact, sim, model


def test_kernel_arithmetic_tracks_the_scheme_on_outliers():
    """With x8 outlier channels the stale max frame and the 2^-4 headroom move the
    result by far less than the scheme's own floor: model ~ simulated oracle to
    0.9995, and model ~ exact within 0.001 of the floor."""
    exact, sim, model = _case(True)
    assert _cos(model, sim) >= 0.9995, _cos(model, sim)
    assert abs(_cos(model, exact) - _cos(sim, exact)) < 1e-3


def test_kernel_arithmetic_tracks_the_scheme_on_normal_inputs():
    exact, sim, model = _case(False)
    assert _cos(model, sim) >= 0.999, _cos(model, sim)
    assert _cos(model, exact) >= 0.995


def test_integer_qk_kernel_arithmetic_meets_the_target_on_outliers():
    """The integer Q.K^T variant's own arithmetic (stale max frame, headroom, V-scale
    fold) on the x8-outlier workload: cosine >= 0.995 against exact attention, the
    target the e4m3 Q.K^T cannot reach there, and close to the int8 simulated oracle."""
    exact, sim, model = _case(True, qk="int8")
    assert _cos(model, exact) >= 0.995, _cos(model, exact)
    assert _cos(model, sim) >= 0.9995, _cos(model, sim)


def test_integer_qk_kernel_arithmetic_on_normal_inputs():
    exact, sim, model = _case(False, qk="int8")
    assert _cos(model, exact) >= 0.995, _cos(model, exact)
    assert _cos(model, sim) >= 0.999, _cos(model, sim)
