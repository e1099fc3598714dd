"""GPU checks of the two FP8 attention variants: the prologue against the
oracle's quantisers, and dit_attn_fp8 (e4m3 Q.K^T) / dit_attn_fp8_i8qk (int8
Q.K^T) against exact fp64 attention and against a float32 model of the
kernels' own arithmetic (tests/fp8_kernel_arith.py).

Bars, and where they come from:

* prologue against the oracle's quantisers: the same codes except where the
  kernel's fp32 rotation and scaling put a value on the other side of a
  rounding point (fewer than 1 in 1000, one step each).  Such a flip in an
  outlier channel of Q moves every score of that row, so the attention kernel
  is compared with the model run on the codes and scales the prologue wrote.
* attention kernel against the model of its arithmetic on those codes, cosine
  >= 0.9999.  The model performs the kernel's steps in the same precisions;
  what it leaves out is the output's single bf16 rounding (relative error <=
  2^-9 per element, which alone keeps the cosine above 1 - 2^-19) and
  ex2.approx / lg2.approx (relative error ~2^-22, so an e4m3 rounding of P
  flips only for values within ~2^-22 of a rounding point: ~2^-18 of the
  elements).  0.9999 leaves those a margin of two orders of magnitude; anything
  that changes the arithmetic (a wrong scale, a lost tile, a misplaced max)
  costs far more.
* against exact attention: the target, cosine >= 0.995, on N(0,1) inputs for
  both variants and on the x8-outlier Flux workloads for the int8 Q.K^T variant.
  On the outlier workloads the e4m3 Q.K^T scheme itself floors near 0.975 (the
  3-bit mantissa on the dominant outlier products; the oracle's simulated
  scheme shows it), so there the e4m3 kernel is held to its model and to that
  floor (model against exact, within 1e-3), not to the target.
"""
import dataclasses
import math

import numpy as np
import pytest
import torch

from conftest import cuda_ok
from fp8_kernel_arith import kernel_model_codes
from oracle import attention as A
from oracle import fp8 as F
from oracle import rope as R
from diffusion_transformer_denoising_dit_b200 import synth
import diffusion_transformer_denoising_dit_b200 as dit

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]
DEV = "cuda"
MODEL_COS = 0.9999
TARGET_COS = 0.995
QK = {"fp8": "e4m3", "fp8_i8qk": "int8"}


def _cos(a, b):
    return float((a * b).sum() / math.sqrt((a * a).sum() * (b * b).sum()))


def _inputs(w, N=None, seed=None):
    q, k, v = synth.qkv(w, device=DEV, N=N, seed=seed)
    Nn = q.shape[2]
    pos = synth.positions(w.T, w.G) if N is None else synth.positions(w.T, int(math.isqrt(max(Nn - w.T, 1))) + 1)[:Nn]
    cos, sin = dit.rope_tables(pos.to(DEV), w.axes, w.theta)
    return q, k, v, pos.numpy(), cos, sin


def _warps(N, picks):
    """Whole aligned 32-row groups (the kernel's warps) starting at the given rows."""
    starts = sorted({min(max(0, p - p % 32), (N - 1) - (N - 1) % 32) for p in picks})
    return np.concatenate([np.arange(s0, min(s0 + 32, N)) for s0 in starts])


def _model_on_kernel_codes(ws, shape, precision, rows, scale=None):
    """The arithmetic model run on the codes and block scales the prologue wrote."""
    B, H, N, d = shape
    vw = dit.fp8_workspace_views(ws, B, H, N, d)
    qk_t = torch.int8 if precision == "fp8_i8qk" else torch.float8_e4m3fn
    q8 = vw["q8"].cpu().view(qk_t).double().numpy()
    k8 = vw["k8"].cpu().view(qk_t).double().numpy()
    v8 = vw["v8"].cpu().view(torch.float8_e4m3fn).double().numpy()
    sc = {n: vw[n].cpu().double().numpy() for n in ("q_scale", "k_scale", "v_scale")}
    return kernel_model_codes(q8, k8, v8, sc["q_scale"], sc["k_scale"], sc["v_scale"], rows, scale=scale,
                              qk=QK[precision])


def _run(w, precision, N=None, seed=None, rows=None, smooth=True):
    q, k, v, pos, cos, sin = _inputs(w, N, seed)
    ws = dit.attention_workspace(*q.shape, precision=precision, device=DEV)
    o = dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws, smooth_k=smooth)
    assert dit.read_error() == 0
    Nn = q.shape[2]
    rows = np.arange(Nn) if rows is None else rows
    args = dict(pos=pos, axes=w.axes, theta=w.theta, rows=rows)
    exact = A.attention(q.cpu(), k.cpu(), v.cpu(), **args)
    mod = _model_on_kernel_codes(ws, q.shape, precision, rows)
    o = o.cpu().double().numpy()[:, :, rows]
    return o, exact, mod


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
@pytest.mark.parametrize("N", [1000, 700])  # 700: the last 128-token slab has no second 64-token block
def test_prologue_matches_oracle_quantiser(precision, N):
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2)
    q, k, v, pos, cos, sin = _inputs(w, N=N, seed=3)
    B, H, N, d = q.shape
    ws = dit.attention_workspace(B, H, N, d, precision=precision, device=DEV)
    dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws)
    views = dit.fp8_workspace_views(ws, B, H, N, d)
    qr = R.apply(q.cpu().double().numpy(), pos, w.axes)
    kr = R.apply(k.cpu().double().numpy(), pos, w.axes)
    mean = kr.mean(axis=2)
    np.testing.assert_allclose(views["k_mean"].cpu().numpy(), mean, rtol=1e-4, atol=1e-4)
    _check_codes(views, precision, qr, F.smooth_k(kr), v.cpu().double().numpy())


def _check_codes(views, precision, q, k_smoothed, v):
    """The prologue's codes and scales against the oracle's quantisers."""
    int8 = precision == "fp8_i8qk"
    for name, x, blk in (("q", q, 128), ("k", k_smoothed, 64), ("v", v, 64)):
        if int8 and name != "v":
            codes, sc = F.quantize_int8_blocks(x, blk)
            got = views[name + "8"].cpu().view(torch.int8).double().numpy()
            step = np.abs(got - codes)
            # fp32 rotation / scaling can land on the other side of a half-integer
            assert (got != codes).mean() < 1e-3 and step.max() <= 1, ((got != codes).mean(), step.max())
        else:
            codes, sc = F.quantize_blocks(x, blk)
            got = views[name + "8"].cpu().view(torch.float8_e4m3fn).double().numpy()
            diff = got != codes
            assert diff.mean() < 1e-3, diff.mean()
            rel = np.abs(got - codes)[diff] / np.maximum(np.abs(codes[diff]), 2.0 ** -6)
            assert (rel <= 0.126).all()
        np.testing.assert_allclose(views[name + "_scale"].cpu().double().numpy(), sc, rtol=2e-5)
    np.testing.assert_allclose(views["v_scale_max"].cpu().numpy(), views["v_scale"].cpu().numpy().max(axis=2))


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
def test_fp8_without_rotary_tables(precision):
    """No rotary tables: the prologue stages no table rows and quantises Q and K
    as given (K still smoothed).  Its codes against the oracle's quantisers on the
    unrotated inputs; the call against the model of the kernel's arithmetic on
    those codes and against exact attention without rotation (B = 2, H = 2,
    N = 700: a ragged last tile)."""
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2, outliers=False)
    q, k, v = synth.qkv(w, device=DEV, N=700, B=2, seed=53)
    B, H, N, d = q.shape
    ws = dit.attention_workspace(B, H, N, d, precision=precision, device=DEV)
    o = dit.attention(q, k, v, None, None, precision=precision, workspace=ws)
    assert dit.read_error() == 0
    views = dit.fp8_workspace_views(ws, B, H, N, d)
    kd = k.cpu().double().numpy()
    np.testing.assert_allclose(views["k_mean"].cpu().numpy(), kd.mean(axis=2), rtol=1e-4, atol=1e-4)
    _check_codes(views, precision, q.cpu().double().numpy(), F.smooth_k(kd), v.cpu().double().numpy())
    rows = np.arange(N)
    exact = A.attention(q.cpu(), k.cpu(), v.cpu())
    mod = _model_on_kernel_codes(ws, q.shape, precision, rows)
    o = o.cpu().double().numpy()
    assert _cos(o, mod) >= MODEL_COS, _cos(o, mod)
    assert _cos(o, exact) >= TARGET_COS, _cos(o, exact)


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
@pytest.mark.parametrize("name,N", [("tiny", None), ("tiny", 129), ("tiny", 1000)])
def test_fp8_tiny_d64_is_unsupported(precision, name, N):
    w = synth.WORKLOADS[name]
    q, k, v, pos, cos, sin = _inputs(w, N)
    with pytest.raises(dit.DitError):
        dit.attention(q, k, v, cos, sin, precision=precision)


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
@pytest.mark.parametrize("N", [1, 64, 65, 129, 700, 4608])
def test_fp8_normal_inputs_meet_target(precision, N):
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2, outliers=False)
    o, exact, mod = _run(w, precision, N=N, seed=N)
    assert _cos(o, exact) >= TARGET_COS, _cos(o, exact)
    assert _cos(o, mod) >= MODEL_COS, _cos(o, mod)


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
def test_fp8_outlier_workload_every_row(precision):
    """The 1024-px outlier workload, two heads, every query row."""
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2)
    o, exact, mod = _run(w, precision)
    assert _cos(o, mod) >= MODEL_COS, _cos(o, mod)
    # No row may drift from the model: a wrong max or a lost tile shows in single
    # rows (cosine near 0).  One e4m3 P code on the other side of a rounding point
    # (rare, see above) moves a near-one-hot row by at most one e4m3 step, 2^-3
    # relative, which keeps its cosine above 0.99.
    per_row = (o * mod).sum(-1) / np.sqrt((o * o).sum(-1) * (mod * mod).sum(-1))
    assert per_row.min() >= 0.99, (per_row.min(), np.unravel_index(per_row.argmin(), per_row.shape))
    if precision == "fp8_i8qk":
        assert _cos(o, exact) >= TARGET_COS, _cos(o, exact)
    else:
        assert _cos(o, exact) >= _cos(mod, exact) - 1e-3, (_cos(o, exact), _cos(mod, exact))


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
def test_fp8_bench_configuration_sampled_rows(precision):
    """The 2048-px benchmark configuration: the first and last warps and random
    warps of every head."""
    w = synth.WORKLOADS["flux2k"]
    picks = [0, w.N - 1] + list(np.random.default_rng(5).integers(0, w.N, 4))
    rows = _warps(w.N, picks)
    o, exact, mod = _run(w, precision, rows=rows)
    assert _cos(o, mod) >= MODEL_COS, _cos(o, mod)
    if precision == "fp8_i8qk":
        assert _cos(o, exact) >= TARGET_COS, _cos(o, exact)
    else:
        assert _cos(o, exact) >= _cos(mod, exact) - 1e-3


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
def test_fp8_smoothing_matters_for_shifted_keys(precision):
    """Keys with a per-channel offset (seeded, N(0, 8^2) per channel; no rotary
    embedding, so the offset stays a per-channel constant): the smoothed call is
    closer to exact attention than the unsmoothed one by at least half the gap the
    model of the kernel's arithmetic shows on the same inputs, and each call
    tracks that model."""
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2, outliers=False)
    q, k, v = synth.qkv(w, device="cpu", N=1024, seed=9)
    g = torch.Generator().manual_seed(19)
    k = (k.float() + 8.0 * torch.randn(1, w.H, 1, w.d, generator=g)).to(torch.bfloat16)
    rows = np.arange(1024)
    exact = A.attention(q, k, v)
    res = {}
    for smooth in (True, False):
        ws = dit.attention_workspace(*q.shape, precision=precision, device=DEV)
        o = dit.attention(q.to(DEV), k.to(DEV), v.to(DEV), precision=precision, smooth_k=smooth, workspace=ws)
        assert dit.read_error() == 0
        o = o.cpu().double().numpy()
        mod = _model_on_kernel_codes(ws, q.shape, precision, rows)
        assert _cos(o, mod) >= MODEL_COS, (smooth, _cos(o, mod))
        res[smooth] = (_cos(o, exact), _cos(mod, exact))
    model_gap = res[True][1] - res[False][1]
    assert model_gap > 0, res
    assert res[True][0] - res[False][0] >= 0.5 * model_gap, res


def test_fp8_calls_on_two_streams_match_serial_calls():
    """The FP8 call launches its prologue passes and the attention kernel as a chain
    of programmatic dependent launches.  Calls of both variants running at the same
    time on two streams (separate inputs and workspaces) give bit for bit what the
    same calls give one after the other, and back-to-back calls on one stream that
    reuse one workspace match them too."""
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=4)
    cases = []
    for seed, precision in ((11, "fp8"), (12, "fp8_i8qk")):
        q, k, v, pos, cos, sin = _inputs(w, N=2048, seed=seed)
        ws = dit.attention_workspace(*q.shape, precision=precision, device=DEV)
        cases.append((q, k, v, cos, sin, precision, ws))
    serial = []
    for q, k, v, cos, sin, precision, ws in cases:
        serial.append(dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws).clone())
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream() for _ in cases]
    outs = []
    torch.cuda.synchronize()
    for (q, k, v, cos, sin, precision, ws), st in zip(cases, streams):
        with torch.cuda.stream(st):
            outs.append([dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws) for _ in range(3)])
    torch.cuda.synchronize()
    assert dit.read_error() == 0
    for ref, got in zip(serial, outs):
        for o in got:
            assert torch.equal(o, ref)


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
@pytest.mark.parametrize("layout", ["bhnd", "bnhd"])
def test_fp8_batched_ragged_and_strided(precision, layout):
    """B = 2, H = 3, N = 700 (a ragged last tile and a last 128-token slab without
    its second 64-token block), in the contiguous [B, H, N, d] layout and in the
    strided [B, N, H, d] one: every row of every (b, h) against the model of the
    kernel's arithmetic on its own codes, and against exact attention."""
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=3, outliers=False)
    N = 700
    q, k, v = synth.qkv(w, device=DEV, N=N, B=2, seed=31)
    if layout == "bnhd":
        q, k, v = (t.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3) for t in (q, k, v))
    pos = synth.positions(w.T, int(math.isqrt(N - w.T)) + 1)[:N]
    cos, sin = dit.rope_tables(pos.to(DEV), w.axes, w.theta)
    ws = dit.attention_workspace(*q.shape, precision=precision, device=DEV)
    o = dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws)
    assert dit.read_error() == 0
    rows = np.arange(N)
    exact = A.attention(q.cpu(), k.cpu(), v.cpu(), pos=pos.numpy(), axes=w.axes, theta=w.theta)
    mod = _model_on_kernel_codes(ws, q.shape, precision, rows)
    o = o.cpu().double().numpy()
    assert _cos(o, mod) >= MODEL_COS, _cos(o, mod)
    assert _cos(o, exact) >= TARGET_COS, _cos(o, exact)
    for b in range(2):  # no (b, h) may be off on its own
        for h in range(3):
            assert _cos(o[b, h], mod[b, h]) >= MODEL_COS, (b, h, _cos(o[b, h], mod[b, h]))


@pytest.mark.parametrize("precision", ["fp8", "fp8_i8qk"])
def test_fp8_explicit_softmax_scale(precision):
    """An explicit softmax scale (0.05 instead of 1/sqrt(d)) reaches both the
    kernel and its model: the call tracks the model run with that scale and exact
    attention with it."""
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2, outliers=False)
    q, k, v, pos, cos, sin = _inputs(w, N=700, seed=41)
    ws = dit.attention_workspace(*q.shape, precision=precision, device=DEV)
    o = dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws, scale=0.05)
    assert dit.read_error() == 0
    rows = np.arange(q.shape[2])
    exact = A.attention(q.cpu(), k.cpu(), v.cpu(), scale=0.05, pos=pos, axes=w.axes, theta=w.theta)
    mod = _model_on_kernel_codes(ws, q.shape, precision, rows, scale=0.05)
    o = o.cpu().double().numpy()
    assert _cos(o, mod) >= MODEL_COS, _cos(o, mod)
    assert _cos(o, exact) >= TARGET_COS, _cos(o, exact)
