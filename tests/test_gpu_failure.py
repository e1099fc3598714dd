"""Failure detection on the GPU without a fault.

Every wait inside the kernels is bounded (1 s of %globaltimer); when it runs out
the kernel records DIT_ERR_TIMEOUT in a device error word and ends normally.
The self-test entry point makes such a wait run out (a barrier nothing arrives
on); the host must read the status, the word must clear on reading, and the
context must stay usable for the next real call.
"""
import math

import numpy as np
import pytest
import torch

from conftest import cuda_ok
from oracle import attention as A
from diffusion_transformer_denoising_dit_b200 import synth
import diffusion_transformer_denoising_dit_b200 as dit

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]
DIT_ERR_TIMEOUT = 6


def test_bounded_wait_times_out_and_context_survives():
    assert dit.read_error() == 0
    dit.selftest_wait_timeout()
    assert dit.read_error() == DIT_ERR_TIMEOUT
    assert dit.read_error() == 0  # cleared by the first read
    # the next real call runs normally on the same context
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv(w, device="cuda")
    pos = synth.positions(w.T, w.G)
    cos, sin = dit.rope_tables(pos.cuda(), w.axes, w.theta)
    o = dit.attention(q, k, v, cos, sin).cpu().double().numpy()
    assert dit.read_error() == 0
    ref = A.attention(q.cpu(), k.cpu(), v.cpu(), pos=pos.numpy(), axes=w.axes, theta=w.theta)
    assert np.abs(o - ref).max() <= 2e-2
    assert float((o * ref).sum() / math.sqrt((o * o).sum() * (ref * ref).sum())) >= 0.9999


def test_timeout_status_is_recorded_once():
    """Two timed-out waits before a read still report one DIT_ERR_TIMEOUT (first error wins)."""
    dit.selftest_wait_timeout()
    dit.selftest_wait_timeout()
    assert dit.read_error() == DIT_ERR_TIMEOUT
    assert dit.read_error() == 0
