"""Pins of the oracle's auxiliary-loss-free bias update.

The pages ("전문가 혼합(Mixture of Experts; MoE)" lesson, "부하 분산 문제" item 3 and
"Step 2: 100개 토큰 라우팅하기") fix the rule's direction (over-used experts -gamma,
under-used +gamma) and its effect: with the update in a loop, the loads of 100 routed
tokens approach the uniform distribution within a few iterations.
"""
import numpy as np

from oracle import moe as M


def test_update_direction_and_exact_fp32_steps():
    # T*k = 40 rows over E = 4 experts: mean 10
    bias = np.array([0.1, -0.25, 0.0, 3.0], dtype=np.float32)
    counts = np.array([11, 9, 10, 10])
    got = M.update_bias(bias, counts, T=20, k=2, gamma=0.01)
    assert got.dtype == np.float32
    exp = np.array([np.float32(0.1) - np.float32(0.01), np.float32(-0.25) + np.float32(0.01),
                    np.float32(0.0), np.float32(3.0)], dtype=np.float32)
    assert np.array_equal(got, exp)


def test_fractional_mean_is_compared_exactly():
    # T*k = 10 rows over E = 3 experts: mean 3.33.., counts 3 / 4 / 3
    got = M.update_bias(np.zeros(3, np.float32), np.array([3, 4, 3]), T=5, k=2, gamma=0.5)
    assert got.tolist() == [0.5, -0.5, 0.5]


def test_gamma_zero_and_balanced_load_leave_bias_unchanged():
    b = np.array([0.3, -0.7], dtype=np.float32)
    assert np.array_equal(M.update_bias(b, np.array([5, 1]), T=3, k=2, gamma=0.0), b)
    assert np.array_equal(M.update_bias(b, np.array([3, 3]), T=3, k=2, gamma=0.1), b)


def _loads(x_bits, W_r, bias, k, E):
    ids, _, _ = M.route(x_bits, W_r, bias, k)
    return np.bincount(ids.ravel(), minlength=E)


def test_update_loop_evens_out_skewed_loads():
    # 100 tokens, 8 experts, top-2, router rows with a strong per-expert preference
    rng = np.random.default_rng(3)
    T, H, E, k = 100, 64, 8, 2
    x = rng.standard_normal((T, H)).astype(np.float32)
    x_bits = (x.view(np.uint32) >> 16).astype(np.uint16)          # bf16 truncation is fine here
    W_r = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    W_r[:, 0] += np.linspace(0.6, -0.6, E).astype(np.float32)     # expert 0 favoured, expert 7 not
    x_bits[:, 0] = np.uint16(0x3F80)                               # channel 0 = 1.0 for every token
    bias = np.zeros(E, np.float32)
    start = _loads(x_bits, W_r, bias, k, E)
    ratios = [start.max() / (T * k / E)]
    for _ in range(50):
        counts = _loads(x_bits, W_r, bias, k, E)
        bias = M.update_bias(bias, counts, T, k, gamma=0.02)
        ratios.append(_loads(x_bits, W_r, bias, k, E).max() / (T * k / E))
    assert ratios[0] > 2.0                      # skewed without the bias
    assert min(ratios[-10:]) < 1.3              # near uniform after the loop
    assert np.mean(ratios[-10:]) < 0.6 * ratios[0]


def test_flipped_sign_would_make_it_worse():
    # the opposite rule (over-used +gamma) drives the load further apart: the pin above
    # distinguishes the two directions
    rng = np.random.default_rng(3)
    T, H, E, k = 100, 64, 8, 2
    x = rng.standard_normal((T, H)).astype(np.float32)
    x_bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    W_r = (rng.standard_normal((E, H)) * 0.05).astype(np.float32)
    W_r[:, 0] += np.linspace(0.6, -0.6, E).astype(np.float32)
    x_bits[:, 0] = np.uint16(0x3F80)
    bias = np.zeros(E, np.float32)
    start = _loads(x_bits, W_r, bias, k, E).max()
    for _ in range(20):
        counts = _loads(x_bits, W_r, bias, k, E)
        bias = M.update_bias(bias, counts, T, k, gamma=-0.02)
    assert _loads(x_bits, W_r, bias, k, E).max() >= start
