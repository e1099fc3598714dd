"""Rotary position embedding, fp64 (oracle; test infrastructure only).

Source: [vflash] "Optimization ledger", table "Accepted or exposed", row
"strict Triton RoPE" names rotary embedding as a separate hot op of DiT
denoising; the axes split (16, 56, 56) of a 128-wide head and theta = 1e4 are
the workload's.  The pages give no formula; this is the textbook rotary
embedding with a multi-axis ("axes") split of the head dimension:

* the head dimension d is split into consecutive axis slices of widths
  (d0, d1, d2), each even;
* inside axis a, channel pair p is (off_a + 2p, off_a + 2p + 1)  -- reading:
  interleaved pairs, the Flux convention;
* that pair is rotated by angle  pos[a] * theta ** (-2p / d_a);
* rotation: y0 = x0 cos(phi) - x1 sin(phi),  y1 = x0 sin(phi) + x1 cos(phi).
"""
from __future__ import annotations

import numpy as np


def angles(pos, axes, theta: float = 10000.0) -> np.ndarray:
    """fp64 [N, d/2] rotation angle of every (token, channel pair).

    pos: integer [N, 3] position ids; axes: (d0, d1, d2) with even widths.
    Pair index is global: axis a's pairs start at off_a / 2.
    """
    pos = np.asarray(pos, dtype=np.float64)
    N = pos.shape[0]
    d = int(sum(axes))
    out = np.zeros((N, d // 2), dtype=np.float64)
    off = 0
    for a, da in enumerate(axes):
        for p in range(da // 2):
            freq = float(theta) ** (-2.0 * p / da)
            out[:, off // 2 + p] = pos[:, a] * freq
        off += da
    return out


def apply(x, pos, axes, theta: float = 10000.0) -> np.ndarray:
    """Rotate x [..., N, d] (any float dtype, upcast to fp64) by the rotary angles."""
    x = np.asarray(x, dtype=np.float64)
    phi = angles(pos, axes, theta)
    c = np.cos(phi)
    s = np.sin(phi)
    x0 = x[..., 0::2]
    x1 = x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y
