"""GPU parity of the rotary-embedding and First-Block-Cache kernels against the fp64 oracle."""
import math

import numpy as np
import pytest
import torch

from conftest import cuda_ok
from oracle import gate as G
from oracle import rope as R
from diffusion_transformer_denoising_dit_b200 import synth
import diffusion_transformer_denoising_dit_b200 as dit

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]
DEV = "cuda"


@pytest.mark.parametrize("name", ["tiny", "flux1k", "flux2k"])
def test_rope_tables_match_oracle_angles(name):
    w = synth.WORKLOADS[name]
    pos = synth.positions(w.T, w.G)
    c, s = dit.rope_tables(pos.to(DEV), w.axes, w.theta)
    ang = R.angles(pos.numpy(), w.axes, w.theta)
    # tables are fp64 values rounded once to fp32: within one fp32 half-ulp of |x| <= 1
    np.testing.assert_allclose(c.cpu().double().numpy(), np.cos(ang), rtol=0, atol=6e-8)
    np.testing.assert_allclose(s.cpu().double().numpy(), np.sin(ang), rtol=0, atol=6e-8)


@pytest.mark.parametrize("name", ["tiny", "flux1k"])
def test_rope_apply_fp32_within_1e3(name):
    w = synth.WORKLOADS[name]
    pos = synth.positions(w.T, w.G)
    q, _, _ = synth.qkv(w, device=DEV)
    c, s = dit.rope_tables(pos.to(DEV), w.axes, w.theta)
    y = dit.rope_apply(q, c, s, out_dtype=torch.float32)
    ref = R.apply(q.cpu().double().numpy(), pos.numpy(), w.axes, w.theta)
    err = np.abs(y.cpu().double().numpy() - ref).max()
    assert err <= 1e-3, err
    assert err <= 1e-4 * max(1.0, np.abs(ref).max())   # what fp32 math actually gives


def test_rope_apply_bench_configuration_sampled_heads():
    """The 2048-px workload at full size (24 heads x 16896 tokens, the bench's K pass in
    fp32 output): every token of the first and last head against the oracle."""
    w = synth.WORKLOADS["flux2k"]
    pos = synth.positions(w.T, w.G)
    q, _, _ = synth.qkv(w, device=DEV)
    c, s = dit.rope_tables(pos.to(DEV), w.axes, w.theta)
    y = dit.rope_apply(q, c, s, out_dtype=torch.float32)
    for h in (0, w.H - 1):
        ref = R.apply(q[:, h].cpu().double().numpy(), pos.numpy(), w.axes, w.theta)
        err = np.abs(y[:, h].cpu().double().numpy() - ref).max()
        assert err <= 1e-3, (h, err)


def test_rope_apply_bf16_within_one_ulp_and_in_place():
    w = synth.WORKLOADS["tiny"]
    pos = synth.positions(w.T, w.G)
    q, _, _ = synth.qkv(w, device=DEV)
    c, s = dit.rope_tables(pos.to(DEV), w.axes, w.theta)
    y = dit.rope_apply(q, c, s)
    ref = torch.from_numpy(R.apply(q.cpu().double().numpy(), pos.numpy(), w.axes, w.theta))
    ref_bf = ref.to(torch.bfloat16).double()
    ulp = torch.where(ref_bf == 0, torch.tensor(2.0 ** -133, dtype=torch.float64),
                      2.0 ** (torch.floor(torch.log2(ref_bf.abs())) - 7))
    assert ((y.cpu().double() - ref_bf).abs() <= ulp).all()
    q2 = q.clone()
    dit.rope_apply(q2, c, s, out=q2)
    assert torch.equal(q2, y)


def test_rope_apply_strided_views():
    """Q laid out [B, N, H, d] (token-major) and viewed as [B, H, N, d]."""
    w = synth.WORKLOADS["tiny"]
    pos = synth.positions(w.T, w.G)
    q, _, _ = synth.qkv(w, device=DEV)
    qt = q.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    c, s = dit.rope_tables(pos.to(DEV), w.axes, w.theta)
    assert torch.equal(dit.rope_apply(qt, c, s), dit.rope_apply(q, c, s))


# ------------------------------------------------------------------ gate
def _gate(cur, prev, thr):
    rel, skip = dit.fbcache_gate(cur.to(DEV), prev.to(DEV), thr)
    return float(rel.item()), int(skip.item())


@pytest.mark.parametrize("eps", [1e-4, 1e-2, 0.3])
def test_gate_eps_sweep_tiny(eps):
    cur, prev = synth.gate_pair(288, 128, eps)
    rel, skip = _gate(cur, prev, 0.08)
    ref = G.relative_l1(cur, prev)
    assert abs(rel - ref) <= 1e-6 * ref + 1e-12
    assert skip == int(G.skip(ref, 0.08))


@pytest.mark.parametrize("thr", [0.08, 0.12, 0.24])
@pytest.mark.parametrize("eps", [1e-4, 1e-2, 0.3])
def test_gate_flux1k_hidden_state(eps, thr):
    cur, prev = synth.gate_pair(4608, 3072, eps, device=DEV)
    rel, skip = _gate(cur, prev, thr)
    ref = G.relative_l1(cur.cpu(), prev.cpu())
    assert abs(rel - ref) <= 1e-5 * ref + 1e-12
    if abs(ref - thr) > 1e-4:
        assert skip == int(G.skip(ref, thr))


@pytest.mark.parametrize("delta", [1e-2, 1e-3, 2e-4, 5e-5, -5e-5, -2e-4, -1e-3, -1e-2])
def test_gate_threshold_band(delta):
    thr = 0.08
    cur, prev = synth.gate_scaled_pair(288, 128, thr + delta)
    rel, skip = _gate(cur, prev, thr)
    ref = G.relative_l1(cur, prev)
    assert abs(rel - ref) <= 1e-6 * ref
    if abs(ref - thr) > 1e-4:
        assert skip == int(G.skip(ref, thr)), (ref, rel)


@pytest.mark.parametrize("n", [1, 7, 8, 9, 2047, 2048, 2049, 123457])
def test_gate_ragged_sizes(n):
    g = torch.Generator().manual_seed(n)
    prev = torch.randn(n, generator=g).to(torch.bfloat16)
    cur = (prev.float() + 0.1 * torch.randn(n, generator=g)).to(torch.bfloat16)
    rel, _ = _gate(cur, prev, 0.1)
    ref = G.relative_l1(cur, prev)
    assert abs(rel - ref) <= 1e-6 * ref + 1e-12


def test_gate_degenerate_cases():
    z = torch.zeros(1000, dtype=torch.bfloat16)
    assert _gate(z, z, 0.08) == (0.0, 1)
    rel, skip = _gate(torch.ones(1000, dtype=torch.bfloat16), z, 0.08)
    assert math.isinf(rel) and skip == 0
    prev = torch.tensor([1.0, -2.0, 0.5, 4.0, 8.0] * 20, dtype=torch.bfloat16)
    assert _gate(prev * 1.125, prev, 0.2) == (0.125, 1)
    assert _gate(-prev, prev, 0.2) == (2.0, 0)


def test_gate_bench_configuration():
    """The bench's residual pair at full size (16896 x 3072 bf16, 51.9 M elements),
    called as the bench calls it, against the fp64 oracle."""
    r_prev, r_cur = synth.gate_pair(16896, 3072, 0.05, seed=4000, device=DEV)
    rel, skip = _gate(r_cur, r_prev, 0.12)
    ref = G.relative_l1(r_cur.cpu(), r_prev.cpu())
    assert abs(rel - ref) <= 1e-5 * ref
    assert abs(ref - 0.12) > 1e-4 and skip == int(G.skip(ref, 0.12))


def test_gate_is_deterministic():
    cur, prev = synth.gate_pair(4608, 3072, 0.05, device=DEV)
    r1, _ = dit.fbcache_gate(cur, prev, 0.1)
    r2, _ = dit.fbcache_gate(cur, prev, 0.1)
    assert r1.item() == r2.item()


def test_gate_trace_decisions_match_oracle():
    """28-step seeded drift at a reduced hidden size: identical skip pattern (16 skipped)."""
    res = list(synth.drift_residuals(1024, 512, steps=28))
    ref = G.trace_decisions(res, 0.12)
    gate = dit.FBCacheGate(0.12, res[0].numel())
    got = [False]
    for t in range(1, 28):
        got.append(bool(gate(res[t].to(DEV), res[t - 1].to(DEV)).item()))
    assert got == [s for _, s in ref]
    assert sum(got) == 16
    assert dit.read_error() == 0


def test_gate_last_computed_policy_matches_oracle():
    """The last-computed policy (compare with the residual of the last step that ran):
    the gate kernel, fed the reference the policy picks, reproduces the oracle's decisions."""
    res = list(synth.drift_residuals(1024, 512, steps=28))
    ref_dec = G.trace_decisions(res, 0.12, policy="last_computed")
    gate = dit.FBCacheGate(0.12, res[0].numel())
    got, ref = [False], 0
    for t in range(1, 28):
        s = bool(gate(res[t].to(DEV), res[ref].to(DEV)).item())
        got.append(s)
        if not s:
            ref = t
    assert got == [s for _, s in ref_dec]
    assert dit.read_error() == 0


@pytest.mark.parametrize("policy", ["consecutive", "last_computed"])
@pytest.mark.parametrize("warmup", [1, 4])
def test_gate_policies_on_the_device_match_oracle(policy, warmup):
    """FBCacheGate.step over the 28-step drift with the reference residual kept on
    the device (no host read inside the loop): the per-step flags equal the
    oracle's decisions under both policies and warm-up lengths."""
    res = [r.to(DEV) for r in synth.drift_residuals(1024, 512, steps=28)]
    ref = G.trace_decisions([r.cpu() for r in res], 0.12, policy=policy, warmup=warmup)
    gate = dit.FBCacheGate(0.12, res[0].numel(), device=DEV, policy=policy, warmup=warmup)
    flags = torch.full((28,), -1, dtype=torch.int32, device=DEV)
    for t in range(28):
        flags[t:t + 1].copy_(gate.step(res[t]))
    got = [bool(x) for x in flags.tolist()]
    assert got == [s for _, s in ref], (got, [s for _, s in ref])
    assert dit.read_error() == 0


@pytest.mark.parametrize("n", [1, 7, 8, 9, 2049, 1000003])
def test_gate_reference_update_follows_the_flag(n):
    """fbcache_gate_ref_update copies r_cur into r_ref exactly when the flag is 0
    (and always without a flag), ragged sizes included."""
    g = torch.Generator(device=DEV).manual_seed(n)
    cur = torch.randn(n, generator=g, device=DEV).to(torch.bfloat16)
    for flag_val, want_copy in ((None, True), (0, True), (1, False)):
        ref = torch.full((n,), 7.0, device=DEV, dtype=torch.bfloat16)
        flag = None if flag_val is None else torch.full((1,), flag_val, dtype=torch.int32, device=DEV)
        dit.fbcache_gate_ref_update(cur, ref, flag)
        torch.cuda.synchronize()
        assert torch.equal(ref, cur) if want_copy else bool((ref == 7.0).all()), (flag_val, n)
    assert dit.read_error() == 0


def test_gate_sums_and_finalize_reproduce_the_gate():
    """fbcache_gate_sums + fbcache_gate_finalize on the whole tensor give fbcache_gate's
    rel bit for bit; from two shards' totals added together, the same decision."""
    for eps in (1e-2, 0.3):
        cur, prev = synth.gate_pair(4608, 3072 // 4, eps, device=DEV)
        rel, skip = dit.fbcache_gate(cur, prev, 0.12)
        rel2, skip2 = dit.fbcache_gate_finalize(dit.fbcache_gate_sums(cur, prev), 0.12)
        assert torch.equal(rel, rel2) and torch.equal(skip, skip2)
        h = cur.shape[0] // 2
        tot = dit.fbcache_gate_sums(cur[:h], prev[:h]) + dit.fbcache_gate_sums(cur[h:], prev[h:])
        rel3, skip3 = dit.fbcache_gate_finalize(tot, 0.12)
        ref = G.relative_l1(cur.cpu(), prev.cpu())
        assert abs(rel3.item() - ref) <= 1e-6 * ref
        assert int(skip3.item()) == int(G.skip(ref, 0.12))
    assert dit.read_error() == 0
