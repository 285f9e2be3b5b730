"""The seeded input recipe: the generators draw what their documentation says,
and the same seed always gives the same bytes (the oracle and the CUDA path
are handed copies of one draw)."""
import math

import torch

import synth


def test_same_seed_same_bytes_other_seed_other_bytes():
    a = synth.gaussian_weights(64, 256, seed=3)
    b = synth.gaussian_weights(64, 256, seed=3)
    c = synth.gaussian_weights(64, 256, seed=4)
    assert torch.equal(a, b) and not torch.equal(a, c)
    assert torch.equal(synth.logstd_weights(8, 512, seed=1), synth.logstd_weights(8, 512, seed=1))
    assert torch.equal(synth.activations(2, 128, seed=5), synth.activations(2, 128, seed=5))


def test_gaussian_weights_std_and_outlier_fraction():
    w = synth.gaussian_weights(1024, 1024, seed=0)
    assert w.dtype == torch.float32 and w.shape == (1024, 1024)
    # without outliers the draw is N(0, 0.02^2)
    base = synth.gaussian_weights(1024, 1024, seed=0, frac=0.0)
    assert abs(base.std().item() - 0.02) < 0.0005
    assert abs(base.mean().item()) < 0.0002
    # the outliers are exactly the base draw times 10, on about 0.1 % of entries
    scaled = w != base
    n = scaled.sum().item()
    expect = 0.001 * w.numel()
    assert abs(n - expect) < 6 * math.sqrt(expect)
    assert torch.allclose(w[scaled], base[scaled] * 10.0)


def test_logstd_weights_group_scales_stay_in_range():
    M, K = 256, 4096
    w = synth.logstd_weights(M, K, seed=2)
    groups = w.reshape(M, K // 32, 32)
    # a group's largest magnitude over its std draw: N(0,1) absmax of 32 is
    # below 5 with overwhelming probability; so absmax / 5 <= std <= 0.05
    amax = groups.abs().amax(dim=2)
    assert amax.max().item() < 5 * 0.05
    # the sample std of the groups spans the log-uniform range [0.005, 0.05]
    s = groups.std(dim=2)
    assert s.min().item() < 0.0065 and s.max().item() > 0.04
    # log-uniform: the median group std sits near the geometric mean
    med = s.median().item()
    assert abs(math.log(med) - 0.5 * (math.log(0.005) + math.log(0.05))) < 0.15


def test_activations_dtype_and_moments():
    for dt in (torch.float16, torch.bfloat16, torch.float32):
        x = synth.activations(4, 8192, seed=9, dtype=dt)
        assert x.dtype == dt and x.shape == (4, 8192)
        xf = x.float()
        assert abs(xf.mean().item()) < 0.03 and abs(xf.std().item() - 1.0) < 0.03
    # the narrow types are the fp32 draw rounded once
    x32 = synth.activations(4, 8192, seed=9, dtype=torch.float32)
    assert torch.equal(synth.activations(4, 8192, seed=9, dtype=torch.float16), x32.half())
