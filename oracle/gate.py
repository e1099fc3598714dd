"""First-Block-Cache gate, fp64 (oracle; test infrastructure only).

Source: [FBCache] paragraph "Add opt-in step caching (First-Block-Cache)": across
denoising steps the first block's residual settles; once it barely changes the
remaining blocks are skipped and their cached output reused, under a threshold
knob ("transformer_cache_threshold").  [VisualGen] calls the same family a
residual-difference threshold (Cache-DiT, 0.24).  The pages give no formula;
readings:

* "barely changes" is measured as the relative L1 difference of the stored
  residuals:  rel = sum|r_t - r_prev| / sum|r_prev|  (equal to mean/mean);
* skip  <=>  rel < threshold (strict);
* sum|r_prev| = 0: rel = 0 if the residuals are identical (skip), else +inf;
* the previous residual is that of the immediately preceding step (block 0
  runs on every step, so it always exists); step 0 is always computed.
"""
from __future__ import annotations

import numpy as np

from .attention import _f64


def relative_l1(r_cur, r_prev) -> float:
    a = _f64(r_cur).ravel()
    b = _f64(r_prev).ravel()
    num = float(np.abs(a - b).sum())
    den = float(np.abs(b).sum())
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


def skip(rel: float, threshold: float) -> bool:
    return rel < threshold


def relative_l1_loops(r_cur, r_prev) -> float:
    """Element-by-element Python loop version, for tiny brute-force checks."""
    a = _f64(r_cur).ravel().tolist()
    b = _f64(r_prev).ravel().tolist()
    num = 0.0
    den = 0.0
    for x, y in zip(a, b):
        num += abs(x - y)
        den += abs(y)
    if den == 0.0:
        return 0.0 if num == 0.0 else float("inf")
    return num / den


def trace_decisions(residuals, threshold: float):
    """Per-step (rel, skip) over a denoising trace; step 0 is always computed."""
    out = [(float("nan"), False)]
    prev = None
    for t, r in enumerate(residuals):
        if t > 0:
            rel = relative_l1(r, prev)
            out.append((rel, skip(rel, threshold)))
        prev = r
    return out
