"""FP8 (e4m3) block quantisation and the simulated-FP8 attention diagnostic (oracle; test infrastructure only).

Sources: [VisualGen] section "why the differences arise" (cuDNN FP8 attention
against VANILLA BF16); [vflash] "Optimization ledger", table "Accepted or
exposed" (SageAttention2, a quantised attention).  The pages name FP8 attention
and a quantised-attention method but give neither the number format nor the
scaling; the readings used here:

* format e4m3 ("fn" variant: bias 7, no infinities, largest finite 448,
  smallest normal 2^-6, subnormal step 2^-9), round to nearest even,
  saturating to +-448;
* per-(batch, head) blocks along the token axis, Q blocks of 128 tokens, K and
  V blocks of 64 tokens, each block scale = amax / 448 (an all-zero block gets
  scale 1);
* K is smoothed before quantisation: the mean over all N tokens of the
  rotated K, per channel, is subtracted.  In exact arithmetic this changes
  every score of row i by the same amount <q_i, mean>, so softmax is unchanged;
* scores s_ij = sigma * sQ(i) * sK(j) * <q8_i, k8_j>;
* P = exp(s - rowmax) is quantised to e4m3 after folding the V block scale in
  (P * 448 * sV(j) / sV_max), and the output is rescaled by sV_max / 448 and
  divided by the row sum of the unquantised P.

An alternative reading of the Q.K^T step, SageAttention's (the quantised
attention the ledger names): Q and K as per-block symmetric int8 (scale
amax / 127, round to nearest even, clipped to +-127) with P.V still in e4m3;
``simulated_attention(..., qk="int8")``.  Pinned by every code, ties, torch's
rounding, the half-step bound, exactness where every step is exact, and an
integer tie that e4m3 breaks.

``simulated_attention`` follows those steps in fp64 on quantised operands.
The scheme is our reading (the pages define none), so it is a diagnostic: it
separates the quantisation floor from kernel errors.  Its implementation of
that reading is pinned by closed forms and invariants (tests): Q = 0 gives the
mean of the dequantised V (with unequal V block scales), one-hot scores give
one dequantised V row, permuting whole K/V blocks changes nothing, V * 2^k
scales O exactly, and a Q block scaled by 2^k equals its rows at 2^k sigma;
each of a list of planted mistakes (a misindexed block scale, the per-head V
maximum replaced, the row sum taken over quantised P, sigma dropped) fails one
of them.  Its row max is the exact one, where a streaming kernel uses a
running max, so it matches a kernel only to within the quantisation noise.
"""
from __future__ import annotations

import math

import numpy as np

from . import rope as _rope
from .attention import _f64

E4M3_MAX = 448.0
_MIN_NORMAL_EXP = -6      # 2^-6 smallest normal
_MANT_BITS = 3


def e4m3_decode(code: int) -> float:
    """Value of an 8-bit e4m3fn code from its bit fields (NaN for S.1111.111)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** _MIN_NORMAL_EXP
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def quantize_e4m3(x) -> np.ndarray:
    """Round x (fp64) to the nearest e4m3 value, ties to even, saturating at +-448."""
    x = np.asarray(x, dtype=np.float64)
    ax = np.abs(x)
    # exponent of the binade holding |x|; below the normal range the spacing is fixed
    with np.errstate(divide="ignore"):
        e = np.floor(np.log2(np.where(ax > 0, ax, 1.0)))
    e = np.maximum(e, _MIN_NORMAL_EXP)
    quantum = np.exp2(e - _MANT_BITS)
    r = np.round(ax / quantum) * quantum        # numpy rounds half to even
    r = np.minimum(r, E4M3_MAX)
    return np.copysign(r, x)


def block_scales(x: np.ndarray, block: int) -> np.ndarray:
    """Per-block amax/448 along axis -2 of x [..., N, d]; all-zero block -> 1."""
    N = x.shape[-2]
    nb = (N + block - 1) // block
    sc = np.empty(x.shape[:-2] + (nb,), dtype=np.float64)
    for i in range(nb):
        a = np.abs(x[..., i * block:(i + 1) * block, :]).max(axis=(-2, -1))
        sc[..., i] = np.where(a > 0, a / E4M3_MAX, 1.0)
    return sc


def quantize_blocks(x: np.ndarray, block: int):
    """(codes as fp64 e4m3 values, scales) for per-block quantisation of x [..., N, d]."""
    sc = block_scales(x, block)
    rep = np.repeat(sc, block, axis=-1)[..., : x.shape[-2]]
    return quantize_e4m3(x / rep[..., None]), sc


INT8_MAX = 127.0


def quantize_int8(x) -> np.ndarray:
    """Symmetric int8: round x (fp64) to the nearest integer, ties to even, clipped to +-127."""
    return np.clip(np.round(np.asarray(x, dtype=np.float64)), -INT8_MAX, INT8_MAX)


def quantize_int8_blocks(x: np.ndarray, block: int):
    """(int8 codes as fp64, scales) for per-block symmetric int8 quantisation of x [..., N, d]:
    each block of `block` tokens of one (batch, head) gets scale amax / 127 (an all-zero
    block gets 1), the reading of SageAttention's 8-bit Q and K."""
    N = x.shape[-2]
    nb = (N + block - 1) // block
    sc = np.empty(x.shape[:-2] + (nb,), dtype=np.float64)
    codes = np.empty_like(x, dtype=np.float64)
    for i in range(nb):
        blk = x[..., i * block:(i + 1) * block, :]
        a = np.abs(blk).max(axis=(-2, -1))
        sc[..., i] = np.where(a > 0, a / INT8_MAX, 1.0)
        codes[..., i * block:(i + 1) * block, :] = quantize_int8(blk / sc[..., i, None, None])
    return codes, sc


def smooth_k(k: np.ndarray) -> np.ndarray:
    """K minus its per-(batch, head) channel mean over all tokens."""
    return k - k.mean(axis=-2, keepdims=True)


def simulated_attention(q, k, v, scale=None, pos=None, axes=None, theta=10000.0,
                        q_block=128, kv_block=64, smooth=True, rows=None, qk="e4m3"):
    """fp64 attention on e4m3-quantised operands (diagnostic of our FP8 reading).

    qk="int8" quantises Q and K to per-block symmetric int8 instead (SageAttention's
    split: 8-bit integer Q.K^T, FP8 P.V); every other step is the same."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    if pos is not None:
        q = _rope.apply(q, pos, axes, theta)
        k = _rope.apply(k, pos, axes, theta)
    if smooth:
        k = smooth_k(k)
    B, H, N, d = q.shape
    sigma = 1.0 / math.sqrt(d) if scale is None or scale <= 0 else float(scale)
    if qk == "e4m3":
        q8, sq = quantize_blocks(q, q_block)
        k8, sk = quantize_blocks(k, kv_block)
    elif qk == "int8":
        q8, sq = quantize_int8_blocks(q, q_block)
        k8, sk = quantize_int8_blocks(k, kv_block)
    else:
        raise ValueError("qk must be 'e4m3' or 'int8'")
    v8, sv = quantize_blocks(v, kv_block)
    ridx = np.arange(N) if rows is None else np.asarray(rows)
    out = np.empty((B, H, len(ridx), d), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            sqr = np.repeat(sq[b, h], q_block)[:N]
            skc = np.repeat(sk[b, h], kv_block)[:N]
            svc = np.repeat(sv[b, h], kv_block)[:N]
            svmax = sv[b, h].max()
            s = sigma * (q8[b, h, ridx] @ k8[b, h].T) * sqr[ridx][:, None] * skc[None, :]
            p = np.exp(s - s.max(axis=1, keepdims=True))
            l = p.sum(axis=1, keepdims=True)
            p8 = quantize_e4m3(p * (E4M3_MAX * svc / svmax)[None, :])
            out[b, h] = (p8 @ v8[b, h]) * (svmax / E4M3_MAX) / l
    return out
