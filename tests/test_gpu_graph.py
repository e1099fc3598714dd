"""The attention calls inside a CUDA graph: captured once with preallocated
outputs and workspaces, replayed, and compared with the same calls made eagerly
(bit for bit).  The FP8 call launches its prologue passes and the attention kernel
as a chain of programmatic dependent launches, which the capture keeps as graph
dependencies."""
import dataclasses
import math

import pytest
import torch

from conftest import cuda_ok
import diffusion_transformer_denoising_dit_b200 as dit
from diffusion_transformer_denoising_dit_b200 import synth

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


@pytest.mark.parametrize("precision", ["bf16", "fp8", "fp8_i8qk"])
def test_attention_replays_from_a_cuda_graph(precision):
    w = dataclasses.replace(synth.WORKLOADS["flux1k"], H=4)
    q, k, v = synth.qkv(w, device="cuda", N=2048, seed=21)
    n = q.shape[2]
    pos = synth.positions(w.T, int(math.isqrt(n - w.T)) + 1)[:n].cuda()
    cos, sin = dit.rope_tables(pos, w.axes, w.theta)
    ws = dit.attention_workspace(*q.shape, precision=precision, device="cuda")
    eager = dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws).clone()
    out = torch.empty_like(q)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream
        dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws, out=out)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    out.zero_()
    with torch.cuda.graph(g):
        dit.attention(q, k, v, cos, sin, precision=precision, workspace=ws, out=out)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, eager)
    assert dit.read_error() == 0
