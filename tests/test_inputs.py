"""The seeded generator: deterministic, chunk-independent, right moments."""
import math

import torch

from latentmoe_expert_routing_b200 import inputs as I


def test_unit_normal_moments_and_range():
    v = I.unit_normal(0, 1, 0, 1 << 20)
    assert abs(v.mean().item()) < 5e-3
    assert abs(v.var().item() - 1.0) < 5e-3
    assert v.abs().max().item() <= 2 * math.sqrt(3.0)


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
