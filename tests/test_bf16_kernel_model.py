"""A float32 model of the BF16 attention kernel's arithmetic, against the oracle (no GPU).

The model follows the kernel's softmax for one warp (32 consecutive rows of a
Q tile) step by step, in fp32 where the kernel computes in fp32:

* operands: the rotated Q and K rounded once to bf16 (as the kernel's tensor-core
  operands are), V in bf16;
* scores per 128-key tile S = Q K^T (exact bf16 products, fp32 sum), scaled by
  scale * log2(e);
* lazy rescale per warp: the running max moves only when some row's tile max
  exceeds it by more than tau (log2 units);
* P = 2^(x - m) in fp32, rounded to bf16 (RNE) for P V; the row sum uses the fp32 P;
* O rescaled by 2^(m_old - m_new) when the max moved; O += P_bf16 V in fp32;
  output O / l rounded once to bf16.

Against exact attention on the same bf16 operands (the oracle's BF16 reading), the
error is the output's own bf16 rounding (half an ulp is 0.0156 for |O| in [4, 8))
plus what bf16 P costs in a stale frame, which grows with tau.  On the warps of
the 1024-px outlier workload below, tau = 8 (the kernel's) stays within the 2e-2
bar and tau = 32 does not (0.0307 at head 22, warp 115; the kernel measured 0.029
there before tau = 8 was chosen).
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention as A
from oracle import rope as R
from diffusion_transformer_denoising_dit_b200 import synth

f32 = np.float32
BAR = 2e-2


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, np.float32)).to(torch.bfloat16).float().numpy()


def kernel_model(q, k, v, pos, axes, theta, rows, tau):
    """q, k, v: [N, d] of one (batch, head); rows: one warp's 32 consecutive rows."""
    qr = A.round_bf16(R.apply(A._f64(q), pos, axes, theta)).astype(f32)
    kr = A.round_bf16(R.apply(A._f64(k), pos, axes, theta)).astype(f32)
    v = A._f64(v).astype(f32)
    N, d = qr.shape
    sl2 = f32(1.0 / math.sqrt(d) * math.log2(math.e))
    m = np.full(len(rows), -np.inf, f32)
    l = np.zeros(len(rows), f32)
    o = np.zeros((len(rows), d), f32)
    for j in range((N + 127) // 128):
        kv0 = j * 128
        s = (qr[rows].astype(np.float64) @ kr[kv0:kv0 + 128].T.astype(np.float64)).astype(f32)
        m_tile = (s * sl2).max(axis=1)
        grow = bool((m_tile > m + f32(tau)).any())
        m_new = np.maximum(m, m_tile) if grow else m
        alpha = np.exp2(m - m_new).astype(f32) if grow else np.ones(len(rows), f32)
        p = np.exp2((s * sl2 - m_new[:, None]).astype(f32)).astype(f32)
        l = (l * alpha + p.sum(axis=1, dtype=f32)).astype(f32)
        if j > 0 and grow:
            o = (o * alpha[:, None]).astype(f32)
        o = (o + (_bf16(p).astype(np.float64) @ v[kv0:kv0 + 128].astype(np.float64)).astype(f32)).astype(f32)
        m = m_new
    return _bf16(o / l[:, None])


@pytest.fixture(scope="module")
def flux1k():
    w = synth.WORKLOADS["flux1k"]
    q, k, v = synth.qkv(w)
    return w, q, k, v, synth.positions(w.T, w.G).numpy()


@pytest.mark.parametrize("head,warp", [(22, 115), (6, 10), (2, 30)])
def test_tau_8_keeps_the_bf16_bar_where_tau_32_breaks_it(flux1k, head, warp):
    w, q, k, v, pos = flux1k
    rows = np.arange(32 * warp, 32 * warp + 32)
    ref = A.attention(q[:, head:head + 1], k[:, head:head + 1], v[:, head:head + 1], pos=pos, axes=w.axes,
                      theta=w.theta, rows=rows, operands="bf16")[0, 0]
    err = {tau: np.abs(kernel_model(q[0, head], k[0, head], v[0, head], pos, w.axes, w.theta, rows, tau) - ref).max()
           for tau in (8, 32)}
    assert err[8] <= BAR < err[32], err
