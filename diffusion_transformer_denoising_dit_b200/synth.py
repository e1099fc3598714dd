"""Seeded synthetic inputs for the DiT joint-attention workloads.

This module only draws numbers and lays out tokens.  It contains none of the
method's arithmetic (no rotation, no softmax, no quantisation, no residual
statistic), so that both the CUDA path and the fp64 oracle can be fed from it
without sharing any computation.

Workloads (named by what they are):

* ``tiny``   -- B=1, H=2, d=64, 32 text + 16x16 image tokens (N=288), RoPE axes
  (16, 24, 24), theta=1e4, Q/K/V ~ N(0, 1).
* ``sdxl``   -- SDXL-like UNet self-attention at 1024 px: B=2 (CFG pair), H=10,
  d=64, N=4096 (64x64 latent grid), no text, no RoPE, Q/K/V ~ N(0, 1)/sqrt(d).
* ``flux1k`` -- Flux-like joint attention at 1024 px: B=1, H=24, d=128,
  512 text + 64x64 image tokens (N=4608), RoPE axes (16, 56, 56), Q/K ~ N(0, 1)
  with 5 % of the channels of each head scaled by 8 (same channels for Q and
  K), V ~ N(0, 1).
* ``flux2k`` -- as ``flux1k`` with a 128x128 image grid (N=16896).

Token order is text first, then the image grid row-major.  Text token t has
position ids (t, 0, 0); image token (r, c) has (0, r, c): a 1-D rotary
embedding over text, a 2-D one over the image (the Flux convention of the
"joint" image+text sequence that the TensorRT-LLM VisualGen page's "DiT"
attention runs over).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    d: int
    T: int           # text tokens
    G: int           # image grid side (G*G image tokens)
    rope: bool
    axes: tuple = (0, 0, 0)
    theta: float = 10000.0
    outliers: bool = False
    prescale: bool = False   # Q/K/V all scaled by 1/sqrt(d) (SDXL-like inputs)
    seed: int = 0

    @property
    def N(self) -> int:
        return self.T + self.G * self.G

    def flops(self) -> float:
        """4*B*H*N^2*d: two N x N x d contractions per (b, h)."""
        return 4.0 * self.B * self.H * self.N * self.N * self.d


WORKLOADS = {
    "tiny": Workload("tiny", 1, 2, 64, 32, 16, True, (16, 24, 24), seed=1000),
    "sdxl": Workload("sdxl", 2, 10, 64, 0, 64, False, prescale=True, seed=1001),
    "flux1k": Workload("flux1k", 1, 24, 128, 512, 64, True, (16, 56, 56),
                       outliers=True, seed=1002),
    "flux2k": Workload("flux2k", 1, 24, 128, 512, 128, True, (16, 56, 56),
                       outliers=True, seed=1003),
}


def positions(T: int, G: int) -> torch.Tensor:
    """int32 [T + G*G, 3] position ids: text (t,0,0), then image (0,r,c)."""
    N = T + G * G
    pos = torch.zeros(N, 3, dtype=torch.int32)
    pos[:T, 0] = torch.arange(T, dtype=torch.int32)
    r = torch.arange(G, dtype=torch.int32).repeat_interleave(G)
    c = torch.arange(G, dtype=torch.int32).repeat(G)
    pos[T:, 1] = r
    pos[T:, 2] = c
    return pos


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def outlier_channels(w: Workload, seed: int | None = None) -> torch.Tensor:
    """bool [H, d]: round(0.05 d) channels per head drawn by a seeded permutation."""
    g = _gen(w.seed + 77 if seed is None else seed, "cpu")
    n_out = int(round(0.05 * w.d))
    mask = torch.zeros(w.H, w.d, dtype=torch.bool)
    for h in range(w.H):
        idx = torch.randperm(w.d, generator=g)[:n_out]
        mask[h, idx] = True
    return mask


def qkv(w: Workload, device="cpu", seed: int | None = None, k_bias: float = 0.0,
        B: int | None = None, N: int | None = None):
    """bf16 Q, K, V of shape [B, H, N, d] (contiguous) for workload ``w``.

    Values are drawn in fp32 then cast to bf16 (round to nearest even).  With
    ``k_bias`` != 0 a constant is added to K on the outlier channels (a
    shifted-key variant that exercises K smoothing).  ``B`` / ``N`` override
    the workload's sizes for small parity cases.
    """
    B = w.B if B is None else B
    N = w.N if N is None else N
    g = _gen(w.seed if seed is None else seed, device)
    shape = (B, w.H, N, w.d)
    q = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    k = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    v = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if w.outliers:
        m = outlier_channels(w).to(device)
        scale = torch.where(m, 8.0, 1.0).to(torch.float32)[None, :, None, :]
        q = q * scale
        k = k * scale
        if k_bias:
            k = k + torch.where(m, float(k_bias), 0.0).to(torch.float32)[None, :, None, :]
    if w.prescale:
        s = 1.0 / math.sqrt(w.d)
        q, k, v = q * s, k * s, v * s
    return (q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16))


def gate_pair(tokens: int, hidden: int, eps: float, seed: int = 2000, device="cpu"):
    """(r_cur, r_prev) bf16 [tokens, hidden]: r_prev ~ N(0,1), r_cur = r_prev + eps*N(0,1)."""
    g = _gen(seed, device)
    prev = torch.randn(tokens, hidden, generator=g, device=device)
    cur = prev + eps * torch.randn(tokens, hidden, generator=g, device=device)
    return cur.to(torch.bfloat16), prev.to(torch.bfloat16)


def gate_scaled_pair(tokens: int, hidden: int, c: float, seed: int = 2100, device="cpu"):
    """(r_cur, r_prev) with r_cur = (1 + c * sign) * r_prev elementwise, sign = +-1 random.

    The relative L1 change of such a pair sits close to |c| (bf16 rounding
    moves it a little); used to place pairs near a threshold.
    """
    g = _gen(seed, device)
    prev = torch.randn(tokens, hidden, generator=g, device=device)
    sgn = torch.where(torch.rand(tokens, hidden, generator=g, device=device) < 0.5, -1.0, 1.0)
    cur = prev * (1.0 + c * sgn)
    return cur.to(torch.bfloat16), prev.to(torch.bfloat16)


def drift_schedule(steps: int = 28, first: float = 0.4, last: float = 0.02):
    """Per-step target relative change delta_k, k = 1..steps-1, geometric from first to last."""
    n = steps - 1
    return [first * (last / first) ** ((k - 1) / (n - 1)) for k in range(1, steps)]


def _smooth_field(tokens: int, hidden: int, g: torch.Generator, device) -> torch.Tensor:
    """Sum of 4 low-frequency sinusoids over (token, channel) with seeded phases."""
    t = torch.arange(tokens, device=device, dtype=torch.float32)[:, None] / tokens
    c = torch.arange(hidden, device=device, dtype=torch.float32)[None, :] / hidden
    u = torch.zeros(tokens, hidden, device=device)
    prm = torch.rand(4, 4, generator=g, device=device)
    for i in range(4):
        ft = 1.0 + 3.0 * prm[i, 0]
        fc = 1.0 + 3.0 * prm[i, 1]
        ph = 2.0 * math.pi * prm[i, 2]
        amp = 0.5 + prm[i, 3]
        u = u + amp * torch.sin(2.0 * math.pi * (ft * t + fc * c) + ph)
    return u


def drift_residuals(tokens: int, hidden: int, steps: int = 28, seed: int = 3000,
                    device="cpu", first: float = 0.4, last: float = 0.02):
    """Yield bf16 block-0 residuals r_0 .. r_{steps-1} drifting by delta_k per step.

    r_0 ~ N(0,1); r_k = r_{k-1} + delta_k * (mean|r_{k-1}| / mean|u_k|) * u_k
    with u_k a smooth seeded field, so that consecutive residuals differ by a
    relative L1 amount close to delta_k.
    """
    g = _gen(seed, device)
    r = torch.randn(tokens, hidden, generator=g, device=device)
    yield r.to(torch.bfloat16)
    for delta in drift_schedule(steps, first, last):
        u = _smooth_field(tokens, hidden, g, device)
        r = r + delta * (r.abs().mean() / u.abs().mean()) * u
        yield r.to(torch.bfloat16)
