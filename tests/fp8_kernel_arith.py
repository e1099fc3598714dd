"""A float32 model of the FP8 attention kernels' arithmetic (test infrastructure).

The model follows the kernel's softmax step by step, in fp32 where the kernel
computes in fp32, on the oracle's 8-bit codes and block scales:

* scores per 128-key tile: S = Q8 K8^T (exact e4m3 or int8 products, fp32 sum),
  scaled per 64-key half by sQ * sK(half) * scale * log2(e);
* lazy rescale per warp of 32 consecutive rows: the running max moves only when
  some row's tile max exceeds it by more than tau = 4 (log2 units);
* P = 2^(x + log2 f - m) with f = sV(half) * 448 / (sV_max * 2^4), rounded to e4m3
  (RNE, saturating) -- the V block scale folded into the exponent;
* row sum of the unrounded P, each half divided by its f (the kernel multiplies
  by an approximate reciprocal, within 2^-22 relative; the model divides), f held
  at or above FLT_MIN as the kernel holds it; O rescaled by
  2^(m_old - m_new) when the max moved; O += P8 V8; output O * sV_max * 2^4 / 448 / l.

Rows are taken in groups of 32 from the start of `rows`: pass whole aligned
32-row blocks for the groups to be the kernel's warps.
"""
import math

import numpy as np

from oracle import attention as A
from oracle import fp8 as F
from oracle import rope as R

f32 = np.float32
TAU = 4
I8_BIAS = 12582912.0  # 1.5 * 2^23: the kernel's integer-to-float bias


def kernel_model(q, k, v, pos, axes, theta, rows, scale=None, qk="e4m3", smooth=True):
    """The model on the oracle's own codes: rotation, smoothing and block
    quantisation in fp64 (oracle.fp8), then kernel_model_codes.
    qk="int8": Q and K as symmetric int8 codes (the integer Q.K^T variant).
    pos None: no rotary embedding; smooth False: K is not mean-smoothed."""
    q, k = A._f64(q), A._f64(k)
    if pos is not None:
        q = R.apply(q, pos, axes, theta)
        k = R.apply(k, pos, axes, theta)
    if smooth:
        k = k - k.mean(axis=-2, keepdims=True)
    v = A._f64(v)
    if qk == "int8":
        q8, sq = F.quantize_int8_blocks(q, 128)
        k8, sk = F.quantize_int8_blocks(k, 64)
    else:
        q8, sq = F.quantize_blocks(q, 128)
        k8, sk = F.quantize_blocks(k, 64)
    v8, sv = F.quantize_blocks(v, 64)
    return kernel_model_codes(q8, k8, v8, sq, sk, sv, rows, scale=scale, qk=qk)


def kernel_model_codes(q8, k8, v8, sq, sk, sv, rows, scale=None, qk="e4m3"):
    """The kernel's softmax and accumulation on given 8-bit codes (values as fp64
    arrays [B, H, N, d]) and block scales (sq [B, H, ceil(N/128)], sk and sv
    [B, H, ceil(N/64)]): e.g. the ones the kernel's own prologue wrote, which
    separates the attention kernel from the prologue's rounding.  The integer
    scores of qk="int8" are exact in fp32 (|S| <= 127^2 * 128 < 2^24)."""
    B, H, N, d = q8.shape
    sigma = 1.0 / math.sqrt(d) if scale is None else scale
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
                        f[sl] = max(f32(sv[b, h][kb]) * vfold, np.finfo(f32).tiny)
                    m_tile = (s * c).max(axis=1)
                    grow = bool((m_tile > m + f32(TAU)).any())
                    m_new = np.maximum(m, m_tile) if grow else m
                    alpha = np.exp2(m - m_new).astype(f32) if grow else np.ones(len(rr), f32)
                    # x = fma(S, c, lf): one rounding; lf = log2 f - m per half, rounded in fp32
                    # as the kernel forms it, and for integer scores (biased by 1.5 * 2^23 in
                    # the kernel) the bias times c comes off lf
                    lf = (np.log2(f)[None, :] - m_new[:, None]).astype(f32)
                    sk_ = s.astype(np.float64)
                    if qk == "int8":
                        lf = (lf - (f32(I8_BIAS) * c).astype(f32)).astype(f32)
                        sk_ = sk_ + I8_BIAS
                    x = (sk_ * c.astype(np.float64) + lf.astype(np.float64)).astype(f32)
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
