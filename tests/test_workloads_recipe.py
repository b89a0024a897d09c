"""The seeded input generators against the recipe they implement (CPU): the
outlier-channel counts and gains, the parameter ranges, the AdaLN modulation's
amplified channels, the weight scale, the tokens per sample and the
algorithmic byte count per element."""
import numpy as np
import torch

import workloads as w


def test_outlier_channels_count_and_gain():
    for name, cfg in w.CONFIGS.items():
        if cfg["dist"] == "adaln":
            continue                      # AdaLN-style gains are continuous
        for d in cfg["d"]:
            for gain in cfg["gains"]:
                g = w.channel_gain(name, d, seed=11, gain=gain)
                assert set(np.unique(g)) <= {1.0, gain}
                assert int((g == gain).sum()) == int(round(cfg["frac"] * d))


def test_adaln_shaped_gain_keeps_its_outliers():
    cfg = w.CONFIGS["pixart_sigma"]
    d = cfg["d"][0]
    base = w.channel_gain("pixart_sigma", d, seed=5, gain=1.0)
    g = w.channel_gain("pixart_sigma", d, seed=5, gain=cfg["gains"][0])
    ratio = g / base
    assert int(np.isclose(ratio, cfg["gains"][0]).sum()) == int(round(cfg["frac"] * d))
    assert np.isclose(np.delete(ratio, np.flatnonzero(np.isclose(ratio, cfg["gains"][0]))), 1.0).all()


def test_parameter_ranges():
    p = w.draw_params(12288, seed=3)
    assert p.shape == (384, 5, 3) and p.dtype == np.float32
    a, b, c = p[..., 0], p[..., 1], p[..., 2]
    assert (a >= -1).all() and (a < 1).all() and (c >= -1).all() and (c < 1).all()
    assert (b >= 0.5).all() and (b <= 2.0).all()      # b = 2^U(-1, 1): never 0
    p16 = w.draw_params16(1152, seed=3)
    assert p16.shape == (72, 4, 3)
    assert (p16[..., 1] >= 0.5).all() and (p16[..., 1] <= 2.0).all()


def test_adaln_modulation_recipe():
    B, d = 3, 1152
    shift, scale = w.draw_adaln(B, d, seed=9)
    assert shift.dtype == torch.bfloat16 and scale.shape == (B, d)
    s = scale.float().numpy()
    n_amp = int(round(0.01 * d))
    for b in range(B):
        big = s[b] >= 5.0
        assert int(big.sum()) == n_amp                  # N(0, 0.5) never reaches 5 here
        assert (s[b][big] <= 30.0).all()
    assert abs(float(shift.float().std()) - 0.5) < 0.05


def test_weight_scale():
    W = w.draw_weight(512, 1024, seed=2)
    assert W.dtype == torch.bfloat16 and W.shape == (512, 1024)
    assert abs(float(W.float().std()) * np.sqrt(1024) - 1.0) < 0.02


def test_tokens_per_sample_cover_every_config():
    assert set(w.TOKENS_PER_SAMPLE) == set(w.CONFIGS)
    for name, cfg in w.CONFIGS.items():
        assert w.TOKENS_PER_SAMPLE[name] >= 1 and cfg["M"] % w.TOKENS_PER_SAMPLE[name] == 0


def test_algorithmic_bytes_per_element():
    # 2 B of bf16 in, half a byte of codes and one scale byte per 32 out.
    assert w.algorithmic_bytes(1, 32) == 32 * 2.53125
    assert w.algorithmic_bytes(16384, 12288) == 16384 * 12288 * 2.53125


def test_cases_are_reproducible():
    c1 = w.make_case("tiny")
    c2 = w.make_case("tiny")
    assert torch.equal(c1.x.view(torch.int16), c2.x.view(torch.int16))
    assert np.array_equal(c1.params, c2.params) and np.array_equal(c1.inv_s, c2.inv_s)
    c3 = w.make_case("tiny", M=64)
    assert torch.equal(c3.x.view(torch.int16), c1.x[:64].view(torch.int16))
