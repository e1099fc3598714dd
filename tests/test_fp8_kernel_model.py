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

f32 = np.float32
TAU = 4


def kernel_model(q, k, v, pos, axes, theta, rows, scale=None):
    q = R.apply(A._f64(q), pos, axes, theta)
    k = R.apply(A._f64(k), pos, axes, theta)
    k = k - k.mean(axis=-2, keepdims=True)
    v = A._f64(v)
    B, H, N, d = q.shape
    sigma = 1.0 / math.sqrt(d) if scale is None else scale
    q8, sq = F.quantize_blocks(q, 128)
    k8, sk = F.quantize_blocks(k, 64)
    v8, sv = F.quantize_blocks(v, 64)
    sl2 = f32(sigma * math.log2(math.e))
    nk, nkv = (N + 63) // 64, (N + 127) // 128
    out = np.empty((B, H, len(rows), d))
    for b in range(B):
        for h in range(H):
            vmax = f32(sv[b, h].max())
            vfold = f32(448.0) / (vmax * f32(2 ** TAU))
            fin = vmax * f32(2 ** TAU) / f32(448.0)
            for w0 in range(0, len(rows), 32):  # one warp: 32 rows
                rr = rows[w0:w0 + 32]
                qs = (sq[b, h][rr // 128].astype(f32) * sl2).astype(f32)
                m = np.full(len(rr), -np.inf, f32)
                l = np.zeros(len(rr), f32)
                o = np.zeros((len(rr), d), f32)
                for j in range(nkv):
                    kv0 = j * 128
                    s = (q8[b, h][rr] @ k8[b, h][kv0:kv0 + 128].T).astype(f32)
                    n = s.shape[1]
                    c = np.empty((len(rr), n), f32)
                    f = np.empty(n, f32)
                    for half in range(2):
                        kb = 2 * j + half
                        if kb >= nk:
                            continue
                        sl = slice(64 * half, min(64 * (half + 1), n))
                        c[:, sl] = qs[:, None] * f32(sk[b, h][kb])
                        f[sl] = f32(sv[b, h][kb]) * vfold
                    m_tile = (s * c).max(axis=1)
                    grow = bool((m_tile > m + f32(TAU)).any())
                    m_new = np.maximum(m, m_tile) if grow else m
                    alpha = np.exp2(m - m_new).astype(f32) if grow else np.ones(len(rr), f32)
                    x = (s * c + (np.log2(f)[None, :] - m_new[:, None])).astype(f32)
                    p = np.exp2(x).astype(f32)
                    p8 = F.quantize_e4m3(p.astype(np.float64))
                    rs = np.zeros(len(rr), f32)
                    for half in range(2):
                        if 64 * half < n:
                            sl = slice(64 * half, min(64 * (half + 1), n))
                            rs = rs + p[:, sl].sum(axis=1, dtype=f32) * (f32(1.0) / f[sl.start])
                    l = (l * alpha + rs).astype(f32)
                    if j > 0 and grow:
                        o = (o * alpha[:, None]).astype(f32)
                    o = (o + (p8 @ v8[b, h][kv0:kv0 + n]).astype(f32)).astype(f32)
                    m = m_new
                out[b, h, w0:w0 + len(rr)] = o * (fin / l)[:, None]
    return out


def _cos(a, b):
    return float((a * b).sum() / math.sqrt((a * a).sum() * (b * b).sum()))


def _case(outliers):
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=2, outliers=outliers)
    q, k, v = synth.qkv(w)
    pos = synth.positions(w.T, w.G).numpy()
    rows = np.unique(np.concatenate([np.arange(0, 128), np.random.default_rng(4).integers(0, w.N, 128)]))
    args = dict(pos=pos, axes=w.axes, theta=w.theta, rows=rows)
    exact = A.attention(q, k, v, **args)
    sim = F.simulated_attention(q, k, v, **args)
    model = kernel_model(q, k, v, pos, w.axes, w.theta, rows)
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
