"""The seeded generator: deterministic, chunk-independent, N(0, 1)."""
import math

import numpy as np
import pytest
import torch
from scipy import stats

from latentmoe_expert_routing_b200 import inputs as I


def test_log_unit_against_libm():
    rng = np.random.RandomState(0)
    u = np.concatenate([rng.uniform(0, 1, 200000), np.arange(1, 4097) * 2.0 ** -32,
                        1 - np.arange(0, 4096) * 2.0 ** -53, [2.0 ** -32, 0.5, 1.0],
                        [math.sqrt(0.5), np.nextafter(math.sqrt(0.5), 1)]])
    got = I.log_unit(torch.from_numpy(u)).numpy()
    ref = np.log(u)
    assert got[-3] == 0.0 and got[-4] == -math.log(2.0)
    ulp = np.abs(got - ref) / np.spacing(np.abs(ref) + (ref == 0))
    assert ulp.max() <= 4


def test_cos_2pi_against_libm_and_quadrants():
    rng = np.random.RandomState(1)
    u = np.concatenate([rng.uniform(0, 1, 200000), np.arange(0, 4096) * 2.0 ** -32,
                        [0.0, 0.125, 0.25, 0.375, 0.5, 0.625, 0.75, 0.875]])
    got = I.cos_2pi(torch.from_numpy(u)).numpy()
    assert np.abs(got - np.cos(2 * np.pi * u)).max() <= 2e-15
    # the quadrant points: exact values where the reduced angle is 0
    assert got[-8:].tolist()[::2] == [1.0, 0.0, -1.0, 0.0]
    assert np.abs(got[-7] - math.sqrt(0.5)) <= 2e-16


def test_sqrt_newton_against_libm():
    rng = np.random.RandomState(2)
    x = np.concatenate([rng.uniform(0, 50, 200000), 2.0 ** rng.uniform(-31, 6, 20000),
                        [0.0, 1.0, 2.0, 0.25, 2.0 ** -31, 44.3614195558365]])
    got = I.sqrt_newton(torch.from_numpy(x)).numpy()
    ref = np.sqrt(x)
    assert [got[-6], got[-5], got[-3]] == [0.0, 1.0, 0.5]        # exact squares
    assert np.max(np.abs(got - ref) / np.spacing(np.maximum(ref, 1e-300))) <= 1


def test_unit_normal_is_standard_normal():
    v = I.unit_normal(0, 1, 0, 1 << 22).numpy()
    assert abs(v.mean()) < 2e-3 and abs(v.var() - 1.0) < 3e-3
    assert stats.kstest(v[:1 << 20], "norm").pvalue > 1e-3
    n = len(v)
    for c in (2.0, 3.0, 4.0):                       # two-sided tail masses
        p = 2 * stats.norm.sf(c)
        got = np.count_nonzero(np.abs(v) > c)
        assert abs(got - n * p) < 6 * math.sqrt(n * p), (c, got, n * p)
    assert np.abs(v).max() <= math.sqrt(-2 * math.log(2.0 ** -32)) + 1e-12


def test_chunking_and_offsets_do_not_change_values():
    a = I.normal_tensor(0, 8, (3000,), 0.5, "bf16", chunk=1000)
    b = I.normal_tensor(0, 8, (3000,), 0.5, "bf16", chunk=1 << 20)
    assert torch.equal(a, b)
    c = I.normal_tensor(0, 8, (1000,), 0.5, "bf16", start=2000)
    assert torch.equal(a[2000:], c)


def test_expert_slices_are_independent_streams():
    cfg = I.CONFIGS["tiny_fp32"]
    allu = I.w_up(cfg)
    assert torch.equal(allu[5], I.w_up(cfg, [5])[0])
    assert not torch.equal(allu[5], allu[6])


def test_outlier_rows():
    cfg = I.CONFIGS["ultra_prefill_bf16"]
    rows = I.outlier_rows(cfg)
    assert len(rows) == 82 and len(set(rows)) == 82
    assert all(0 <= r < cfg.T for r in rows)
    x = I.hidden(cfg.replace(D=256), T=512)
    big = [r for r in rows if r < 512]
    rms = x.float().pow(2).mean(1).sqrt()
    assert all(rms[r] > 4 for r in big)
    assert rms[[r for r in range(512) if r not in big]].max() < 1.5


def test_row_window_matches_full_tensor():
    cfg = I.CONFIGS["ultra_prefill_bf16"].replace(D=256)
    full = I.hidden(cfg, T=300)
    part = I.hidden(cfg, T=100, start_row=150)
    assert torch.equal(full[150:250], part)


def test_zipf_bias_profile():
    b = I.gate_bias(I.CONFIGS["skewed_prefill_w4a4"]).double()
    p = torch.exp(2 * b)
    assert abs(p.sum().item() - 1) < 1e-5
    assert abs(p[0].item() / p[1].item() - 2 ** 1.1) < 1e-4


def test_bias_spread_readings():
    """N(0, 0.01) read as a variance (std 0.1, the decode workload) and as a
    standard deviation (0.01, its companion): the same draws, scaled."""
    b1 = I.gate_bias(I.CONFIGS["ultra_decode_bf16"]).double()
    b2 = I.gate_bias(I.CONFIGS["ultra_decode_bf16_bias_sd001"]).double()
    assert 0.085 < b1.std().item() < 0.115 and 0.0085 < b2.std().item() < 0.0115
    assert torch.allclose(b2, 0.1 * b1, rtol=0, atol=1e-8)


@pytest.mark.gpu
def test_generator_bit_identical_on_gpu():
    """The CPU oracle and the GPU path read the same tensors when each
    generates them on its own device."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    a = I.unit_normal(0, 9, (1 << 33) - 5000, 1 << 20)
    b = I.unit_normal(0, 9, (1 << 33) - 5000, 1 << 20, device="cuda").cpu()
    assert torch.equal(a.view(torch.int64), b.view(torch.int64))
    cfg = I.CONFIGS["tiny_fp32"].replace(dtype="bf16", D=512, L=256, F=512, Fs=512)
    for f in (I.w_gate, I.w_fc1, I.w_shared_down, I.hidden):
        assert torch.equal(f(cfg).view(torch.int16), f(cfg, "cuda").cpu().view(torch.int16))
    assert torch.equal(I.w_up(cfg, [3]).view(torch.int16),
                       I.w_up(cfg, [3], device="cuda").cpu().view(torch.int16))
