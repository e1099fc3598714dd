"""The sequence-parallel wrapper on the GPU, one rank (an NCCL group of one):
the exchanges are identities there, so the result must equal the plain call bit
for bit, through this library's kernels.  Layout and exchanges across two ranks
are covered on the CPU (tests/test_multirank.py); more GPUs are not available
to these tests."""
import os
import socket

import pytest
import torch

from conftest import cuda_ok
from diffusion_transformer_denoising_dit_b200 import synth, ulysses
import diffusion_transformer_denoising_dit_b200 as dit

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


@pytest.fixture(scope="module")
def group():
    import datetime
    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    yield None
    dist.destroy_process_group()


def test_one_rank_ulysses_equals_the_plain_call(group):
    w = synth.WORKLOADS["flux1k"]
    q, k, v = synth.qkv(w, device="cuda")
    pos = synth.positions(w.T, w.G)
    cos, sin = dit.rope_tables(pos.cuda(), w.axes, w.theta)
    ref = dit.attention(q, k, v, cos, sin)
    got = ulysses.attention(q, k, v, cos, sin)
    assert torch.equal(got, ref)
    for chunks in (2, 4):  # head chunks overlapped with the exchanges: the same kernels per head
        assert torch.equal(ulysses.attention_overlapped(q, k, v, cos, sin, chunks=chunks), ref)
    cur, prev = synth.gate_pair(4608, 768, 0.05, device="cuda")
    rel, skip = ulysses.gate(cur, prev, 0.12)
    rel_ref, skip_ref = dit.fbcache_gate(cur, prev, 0.12)
    assert torch.equal(rel, rel_ref) and torch.equal(skip, skip_ref)
    assert dit.read_error() == 0
