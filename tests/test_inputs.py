"""Checks on the seeded workload generators (shapes, determinism, skew)."""
import numpy as np
import torch

from fp8_fp4_moe_b200 import inputs as I
from oracle import calibrate_zipf, formats as F


def test_generators_are_deterministic_and_shaped():
    w = I.WORKLOADS["tiny"]
    a = I.make_inputs(w, seed=0)
    b = I.make_inputs(w, seed=0)
    c = I.make_inputs(w, seed=1)
    for key in a:
        assert torch.equal(a[key], b[key])
    assert not torch.equal(a["x"], c["x"])
    assert a["W1"].shape == (8, 1024, 128) and a["W1_scales"].shape == (8, 1024, 8)
    assert a["W2"].shape == (8, 256, 256) and a["W2_scales"].shape == (8, 256, 16)


def test_fixture_mxfp4_weights_approximate_their_draw():
    # the fixture quantiser maps N(0, 0.02) onto MXFP4 with at most half an
    # E2M1 step of error per element relative to the block scale
    w = I.Workload("q", T=1, H=256, I=128, E=1, k=1, shared=0, router_std=0.01, bias="zeros")
    g = I._gen(0, 100, 0, 1)
    raw = torch.randn(2 * w.I, w.H, generator=g) * w.weight_std
    W1, W1s, _, _ = I.make_expert_weights(w, seed=0)
    deq = F.dequant_mxfp4(W1[0].numpy(), W1s[0].numpy())
    scale = np.repeat(F.decode_ue8m0(W1s[0].numpy()), 32, axis=-1)
    assert np.all(np.abs(deq - raw.double().numpy()) <= scale * 1.0 + 1e-12)
    assert np.all(np.abs(raw.double().numpy()) <= 6 * scale + 1e-12)


def test_zipf_constant_gives_about_ten_times_mean_load():
    w = I.WORKLOADS["dsv3_t8192_zipf"]
    x, W_r, _ = I.make_routing_inputs(w, 0)
    from oracle import moe as M
    s = M.router_scores(x.view(torch.int16).numpy().view(np.uint16), W_r.numpy())
    r = calibrate_zipf.max_load_ratio(w, s, I.ZIPF_BETA_T8192)
    assert 9.5 <= r <= 10.5
