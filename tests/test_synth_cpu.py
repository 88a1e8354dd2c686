"""The seeded input recipes hold what the documentation states: the same seed
gives the same bytes, the activations are Student-t with nu = 3 plus eight
outlier channels x200 on a seeded permutation, weights are N(0, sigma), the
decay-gate parameters fall in their stated ranges, and the fused projection
widths are the ones the workloads name."""
import math

import numpy as np
import pytest
import torch
from scipy import stats

from nvfp4_w4a4_quantized_09_b200 import synth


def test_same_seed_same_bytes_other_seed_other_bytes():
    a = synth.student_t_activations(64, 256, seed=7)
    b = synth.student_t_activations(64, 256, seed=7)
    c = synth.student_t_activations(64, 256, seed=8)
    assert a.dtype == torch.bfloat16 and a.shape == (64, 256)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert not torch.equal(a.view(torch.int16), c.view(torch.int16))
    w1 = synth.gaussian_weights(32, 64, 0.02, seed=3)
    w2 = synth.gaussian_weights(32, 64, 0.02, seed=3)
    assert torch.equal(w1.view(torch.int16), w2.view(torch.int16))


def test_outlier_channels_are_the_seeded_permutation_times_200():
    rows, cols = 2048, 512
    x = synth.student_t_activations(rows, cols, seed=11).float()
    ch = torch.randperm(cols, generator=torch.Generator().manual_seed(2))[:8]
    med = x.abs().median(dim=0).values
    mask = torch.zeros(cols, dtype=torch.bool)
    mask[ch] = True
    ratio = float(med[mask].median() / med[~mask].median())
    assert 170 < ratio < 235, ratio                    # medians of |x|: 200 up to sampling noise
    # exactly those eight columns stand out
    assert set(torch.topk(med, 8).indices.tolist()) == set(ch.tolist())


def test_activation_body_is_student_t_nu3():
    x = synth.student_t_activations(1024, 1024, seed=5, n_outliers=0).float().numpy().ravel()
    # Kolmogorov-Smirnov against the library's t distribution (BF16 rounding is
    # far below the statistic's resolution at this sample size)
    d, p = stats.kstest(x, stats.t(df=3).cdf)
    assert d < 0.003, (d, p)
    # the tail that makes the global scale outlier-driven
    tail = float(np.mean(np.abs(x) > 10.0))
    want = 2 * stats.t(df=3).sf(10.0)
    assert abs(tail - want) < 0.2 * want, (tail, want)


@pytest.mark.parametrize("sigma", [0.2, 0.015, 0.002])
def test_weights_are_gaussian_with_the_module_sigma(sigma):
    w = synth.gaussian_weights(512, 1024, sigma, seed=21).float().numpy().ravel()
    assert abs(w.std() / sigma - 1.0) < 0.01
    assert abs(w.mean()) < 4 * sigma / math.sqrt(w.size)
    d, _ = stats.kstest(w / sigma, stats.norm.cdf)
    assert d < 0.01


def test_tiny_inputs_are_rounded_once_and_carry_one_percent_outliers():
    xb, wb, x, w = synth.tiny_inputs()
    assert xb.shape == (64, 256) and wb.shape == (128, 256)
    assert torch.equal(xb.view(torch.int16), x.to(torch.bfloat16).view(torch.int16))
    assert torch.equal(wb.view(torch.int16), w.to(torch.bfloat16).view(torch.int16))
    big = float((x.abs() > 6.0).float().mean())       # N(0,1) alone: 2e-9; x50 entries: ~0.9 %
    assert 0.004 < big < 0.016, big


def test_gate_parameters_in_their_stated_ranges():
    a_log, dt_bias = synth.gdn_gate_params(4096, seed=40)
    assert a_log.dtype == torch.float32 and dt_bias.dtype == torch.float32
    A = torch.exp(a_log.double())
    assert float(A.min()) >= 1.0 - 1e-6 and float(A.max()) <= 16.0 + 1e-5
    dt = torch.nn.functional.softplus(dt_bias.double())
    assert float(dt.min()) >= 1e-3 * (1 - 1e-5) and float(dt.max()) <= 1e-1 * (1 + 1e-5)
    # log-uniform: log dt spread evenly over [log 1e-3, log 1e-1]
    u = (torch.log(dt) - math.log(1e-3)) / (math.log(1e-1) - math.log(1e-3))
    d, _ = stats.kstest(u.numpy(), stats.uniform.cdf)
    assert d < 0.03


def test_fused_projection_widths():
    assert sum(n for _, n, _ in synth.GDN_MODULES) == 24704
    assert sum(n for _, n, _ in synth.GDN_MODULES_DECODE) == 24640
    assert [m for m, _, _ in synth.GDN_MODULES] == ["q", "k", "v", "z", "b", "a"]
    assert synth.MLP_WIDTH * 2 == 34816 and synth.HIDDEN == 5120
