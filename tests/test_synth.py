"""The seeded input generators follow the stated recipe (no GPU).

These inputs feed both the CUDA path and the oracle, so a wrong recipe would
go unnoticed by parity: the checks here hold it to the workloads' stated
shapes, token layout, distributions and seeds.
"""
import math

import pytest
import torch

from diffusion_transformer_denoising_dit_b200 import synth

W = synth.WORKLOADS


def test_workload_sizes_and_flops():
    assert (W["tiny"].N, W["sdxl"].N, W["flux1k"].N, W["flux2k"].N) == (288, 4096, 4608, 16896)
    assert W["flux2k"].flops() == 4 * 24 * 16896 ** 2 * 128
    assert abs(W["flux2k"].flops() - 3.5079e12) < 1e8
    assert W["tiny"].axes == (16, 24, 24) and sum(W["tiny"].axes) == W["tiny"].d
    assert W["flux2k"].axes == (16, 56, 56) and sum(W["flux2k"].axes) == W["flux2k"].d
    assert [W[n].seed for n in ("tiny", "sdxl", "flux1k", "flux2k")] == [1000, 1001, 1002, 1003]


def test_positions_text_then_row_major_image():
    pos = synth.positions(3, 4)
    assert pos.dtype == torch.int32 and tuple(pos.shape) == (3 + 16, 3)
    assert pos[:3].tolist() == [[0, 0, 0], [1, 0, 0], [2, 0, 0]]
    img = pos[3:].tolist()
    assert img == [[0, r, c] for r in range(4) for c in range(4)]


def test_outlier_channels_six_per_head_shared_by_q_and_k():
    w = W["flux1k"]
    m = synth.outlier_channels(w)
    assert tuple(m.shape) == (24, 128)
    assert (m.sum(dim=1) == round(0.05 * 128)).all()
    assert torch.equal(m, synth.outlier_channels(w))                # seeded
    assert not all(torch.equal(m[0], m[h]) for h in range(1, 24))   # drawn per head
    q, k, v = synth.qkv(w, N=2048)
    for t, scaled in ((q, True), (k, True), (v, False)):
        sd = t.float().std(dim=2)[0]                                 # [H, d] over tokens
        out, rest = sd[m], sd[~m]
        assert abs(rest.mean().item() - 1.0) < 0.05
        if scaled:
            assert abs(out.mean().item() - 8.0) < 0.4
        else:
            assert abs(out.mean().item() - 1.0) < 0.05


def test_sdxl_inputs_are_prescaled_without_text_or_rope():
    w = W["sdxl"]
    assert not w.rope and w.T == 0 and w.prescale
    q, k, v = synth.qkv(w, N=512)
    for t in (q, k, v):
        assert tuple(t.shape) == (2, 10, 512, 64)
        assert abs(t.float().std().item() - 1.0 / math.sqrt(64)) < 0.005


def test_qkv_bf16_contiguous_seeded():
    w = W["tiny"]
    a = synth.qkv(w)
    b = synth.qkv(w)
    c = synth.qkv(w, seed=5)
    for x, y, z in zip(a, b, c):
        assert x.dtype == torch.bfloat16 and x.is_contiguous() and tuple(x.shape) == (1, 2, 288, 64)
        assert torch.equal(x, y) and not torch.equal(x, z)
    assert not torch.equal(a[0], a[1])   # Q, K, V are distinct draws


def test_gate_pairs():
    cur, prev = synth.gate_pair(64, 32, 0.0)
    assert torch.equal(cur, prev)
    cur, prev = synth.gate_scaled_pair(64, 32, 0.25)
    ratio = (cur.double() / prev.double()).flatten()
    assert ((ratio - 1.25).abs() < 1e-2).float().mean() > 0.4
    assert ((ratio - 0.75).abs() < 1e-2).float().mean() > 0.4


def test_drift_schedule_is_geometric_and_straddles_the_threshold():
    d = synth.drift_schedule(28)
    assert len(d) == 27
    assert d[0] == pytest.approx(0.4) and d[-1] == pytest.approx(0.02)
    ratios = [d[i + 1] / d[i] for i in range(26)]
    assert max(ratios) - min(ratios) < 1e-12
    # delta_11 = 0.1264 computes, delta_12 = 0.1126 skips at threshold 0.12: 16 skipped steps
    assert d[10] == pytest.approx(0.1264, abs=1e-4) and d[11] == pytest.approx(0.1126, abs=1e-4)
    assert sum(x < 0.12 for x in d) == 16
    assert min(abs(x - 0.12) for x in d) > 6e-3
