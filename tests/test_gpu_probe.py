"""The unit-rate probe (dit_probe_unit_rates) on the GPU: the rates the attention
rooflines are drawn against come out in the ranges a B200 SM has (dense tensor
FLOP per clock per SM: 8192 bf16 and 16384 e4m3 nominal; 16 ex2 results per
clock per SM), and the e4m3 MMA rate is twice the bf16 one."""
import pytest

from conftest import cuda_ok
import diffusion_transformer_denoising_dit_b200 as dit

pytestmark = [pytest.mark.gpu, pytest.mark.skipif(not cuda_ok(), reason="needs a CUDA GPU")]


def test_unit_rates_are_plausible():
    r = dit.probe_unit_rates()
    assert dit.read_error() == 0
    assert 4000 <= r["mma_bf16_flop"] <= 8200, r
    assert 1.9 <= r["mma_e4m3_flop"] / r["mma_bf16_flop"] <= 2.1, r
    assert 8 <= r["ex2_results"] <= 33, r
    assert r["cvt_e4m3x2_instructions"] > 4, r
