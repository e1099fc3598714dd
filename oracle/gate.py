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

Policy variants (the pages name the knob, not the policy): "consecutive" (the
reading above) and "last_computed", where a step is compared with the residual
of the last step whose remaining blocks actually ran (the step the cached
output belongs to), so that small changes accumulate across skipped steps; and
a warm-up of steps that are always computed ([FBCache] and [vflash] both
describe early denoising steps as the ones that must run).
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


def trace_decisions(residuals, threshold: float, policy: str = "consecutive", warmup: int = 1):
    """Per-step (rel, skip) over a denoising trace.

    policy "consecutive": step t is compared with step t-1; "last_computed": with
    the last step that was not skipped.  The first max(warmup, 1) steps are always
    computed (their rel is still reported from step 1 on).
    """
    if policy not in ("consecutive", "last_computed"):
        raise ValueError(policy)
    out = []
    ref = None  # index of the residual step t is compared with
    for t, r in enumerate(residuals):
        if t == 0:
            out.append((float("nan"), False))
            ref = 0
            continue
        base = t - 1 if policy == "consecutive" else ref
        rel = relative_l1(r, residuals[base])
        s = skip(rel, threshold) and t >= warmup
        out.append((rel, s))
        if not s:
            ref = t
    return out
