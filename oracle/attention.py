"""Exact joint image+text multi-head self-attention, fp64 (oracle; test infrastructure only).

Source: [VisualGen] section "why the differences arise": the DiT's VANILLA BF16
attention (about 60 % of the DiT's GPU kernel time) runs over the joint
text+image token sequence, bidirectionally.  The pages print no formula; the
operation the name denotes is scaled dot-product attention

    s_ij = sigma * <R_i q_i, R_j k_j>,     sigma = 1/sqrt(d) unless given
    O_i  = sum_j exp(s_ij - max_j s_ij) v_j / sum_j exp(s_ij - max_j s_ij)

over every key j of the same (batch, head): no mask, no dropout, forward only
(the pages are about inference).  R_i is the rotary embedding of token i
(``oracle.rope``), applied to Q and K but not to V; without position ids it is
the identity.
"""
from __future__ import annotations

import math

import numpy as np

from . import rope as _rope


def round_bf16(x) -> np.ndarray:
    """Round fp64 values to the nearest bfloat16 (8 significant bits), ties to even.

    bfloat16 keeps float32's exponent range and 7 stored mantissa bits; the
    values met here are normal, so the spacing in binade [2^e, 2^(e+1)) is
    2^(e-7).  Zero stays zero.
    """
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, -126.0)
    q = np.exp2(e - 7)
    return np.copysign(np.round(ax / q) * q, x)


def _f64(t) -> np.ndarray:
    """Exact fp64 copy of a tensor/array (bf16 values upcast exactly)."""
    try:
        import torch
        if isinstance(t, torch.Tensor):
            return t.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(t, dtype=np.float64)


def rotate(x, pos, axes, theta):
    """Q or K after rotary embedding (identity when pos is None)."""
    x = _f64(x)
    if pos is None:
        return x
    return _rope.apply(x, pos, axes, theta)


def attention(q, k, v, scale=None, pos=None, axes=None, theta=10000.0,
              rows=None, chunk=1024, operands=None) -> np.ndarray:
    """fp64 O for q, k, v of shape [B, H, N, d].

    rows: optional 1-D index array of query rows to evaluate (same for every
    (b, h)); the result then has shape [B, H, len(rows), d].
    operands: None keeps the rotated Q and K exact; "bf16" rounds them once to
    bfloat16, the reading of the BF16 variant (its tensor-core operands are the
    rotated Q and K as bf16 tensors, as when a RoPE kernel writes bf16 that a
    BF16 attention kernel reads).  Without rotation the inputs are bf16 already.
    """
    q = rotate(q, pos, axes, theta)
    k = rotate(k, pos, axes, theta)
    if operands == "bf16":
        q = round_bf16(q)
        k = round_bf16(k)
    elif operands is not None:
        raise ValueError("operands must be None or 'bf16'")
    v = _f64(v)
    B, H, N, d = q.shape
    sigma = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else float(scale)
    ridx = np.arange(N) if rows is None else np.asarray(rows)
    out = np.empty((B, H, len(ridx), d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            kt = k[b, h].T
            for r0 in range(0, len(ridx), chunk):
                sel = ridx[r0:r0 + chunk]
                s = sigma * (q[b, h, sel] @ kt)           # [r, N]
                s = s - s.max(axis=1, keepdims=True)
                e = np.exp(s)
                out[b, h, r0:r0 + len(sel)] = (e @ v[b, h]) / e.sum(axis=1, keepdims=True)
    return out


def attention_loops(q, k, v, scale=None):
    """Pure-Python triple loop version (no RoPE) for tiny brute-force checks."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, N, d = q.shape
    sigma = 1.0 / math.sqrt(d) if scale is None else float(scale)
    out = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            for i in range(N):
                s = [sigma * sum(q[b, h, i, c] * k[b, h, j, c] for c in range(d)) for j in range(N)]
                m = max(s)
                w = [math.exp(x - m) for x in s]
                z = sum(w)
                for c in range(d):
                    out[b, h, i, c] = sum(w[j] * v[b, h, j, c] for j in range(N)) / z
    return out
