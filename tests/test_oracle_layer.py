"""Pins for the oracle's whole-layer forward.

* a hand-worked 1-token / 4-expert layer whose every intermediate follows in
  closed form from the format definitions (derivation in the comments);
* k = E reducing to the dense gate-weighted sum over all experts;
* identical experts reducing to one expert;
* invariance to the token order;
* doubling every W2 scale doubling the output exactly;
* the activation quantiser against an independent E4M3 codec.
"""
import math

import ml_dtypes
import numpy as np
import pytest
import torch

from fp8_fp4_moe_b200 import inputs as I
from oracle import formats as F
from oracle import moe as M

E2M1_CODE = {0.0: 0, 0.5: 1, 1.0: 2, 1.5: 3, 2.0: 4, 3.0: 5, 4.0: 6, 6.0: 7}


def _e2m1(v):
    return E2M1_CODE[abs(v)] | (8 if v < 0 else 0)


def _bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _hand_layer(bias, shared_expert=False):
    """T=1, H=I=128, E=4, k=2.  x0=1, x1=2; expert e has only
    W1[e][0][0]=a, W1[e][I][1]=b, W2[e][0][0]=c, W2[e][1][0]=d (scales 2^0)."""
    H = Ii = 128
    E = 4
    params = [(1, 1, 1, 1), (-1, 2, 0.5, 1), (1, 0.5, 2, -1), (2, 1, 1, -0.5)]
    if shared_expert:
        params.append((1, 1, 1, 1))
    n = len(params)
    x = np.zeros((1, H), dtype=np.float32)
    x[0, 0], x[0, 1] = 1.0, 2.0
    Wr = np.zeros((E, H), dtype=np.float32)
    Wr[0, 0] = 0.5
    Wr[1, 1] = 0.5
    Wr[2, 0] = 0.25
    Wr[3, 0] = Wr[3, 1] = 0.5
    W1 = np.zeros((n, 2 * Ii, H // 2), dtype=np.uint8)
    W2 = np.zeros((n, H, Ii // 2), dtype=np.uint8)
    for e, (a, b, c, d) in enumerate(params):
        W1[e, 0, 0] = _e2m1(a)               # element 0 -> low nibble
        W1[e, Ii, 0] = _e2m1(b) << 4         # element 1 -> high nibble
        W2[e, 0, 0] = _e2m1(c)
        W2[e, 1, 0] = _e2m1(d)
    W1s = np.full((n, 2 * Ii, H // 32), 127, dtype=np.uint8)
    W2s = np.full((n, H, Ii // 32), 127, dtype=np.uint8)
    return _bf16_bits(x), Wr, np.asarray(bias, np.float32), W1, W1s, W2, W2s


def _silu(z):
    return z / (1 + math.exp(-z))


# Per expert, h0 = silu(a) * (2b) (x is exact after quantisation: amax 2 -> p=-7,
# codes 128 and 256).  Requantised with the smallest 2^p >= |h0|/448 and E4M3 RNE:
#   e0: silu(1)*2   = 1.46212 -> p=-8, 374.3 -> 384 -> 1.5
#   e1: silu(-1)*4  = -1.07577 -> p=-8, -275.4 -> -288 -> -1.125
#   e2: silu(1)*1   = 0.73106 -> p=-9, 374.3 -> 384 -> 0.75
#   e3: silu(2)*2   = 3.52319 -> p=-6, 225.5 -> 224 -> 3.5
# Expert rows (o0, o1) = (hq*c, hq*d), exact in bf16.
HQ = {0: 1.5, 1: -1.125, 2: 0.75, 3: 3.5}
ROWS = {0: (1.5, 1.5), 1: (-0.5625, -1.125), 2: (1.5, -0.75), 3: (3.5, -1.75)}
H0 = {0: _silu(1) * 2, 1: _silu(-1) * 4, 2: _silu(1) * 1, 3: _silu(2) * 2}


@pytest.mark.parametrize("bias,ids,sel_scores,out01", [
    ([0, 0, 1, 0], [3, 2], (1.5, 0.25), (3.046875, -1.5234375)),
    ([0, 0, 0, 0], [3, 1], (1.5, 1.0), (1.96875, -1.515625)),
    ([0, 0.5, 0, 0], [1, 3], (1.0, 1.5), (1.96875, -1.515625)),   # exact tie 1.5 == 1.5
])
def test_hand_worked_single_token(bias, ids, sel_scores, out01):
    xb, Wr, b, W1, W1s, W2, W2s = _hand_layer(bias)
    r = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=2, shared=0, keep_rows=True)
    assert r["scores"][0].tolist() == [0.5, 1.0, 0.25, 1.5]
    assert r["ids"][0].tolist() == ids
    e0, e1 = (math.exp(v) for v in sel_scores)
    g = [e0 / (e0 + e1), e1 / (e0 + e1)]
    assert r["gates"][0] == pytest.approx(g, abs=1e-15)
    for e in ids:
        lst, res = r["rows"][e]
        assert res["h"][0, 0] == pytest.approx(H0[e], rel=1e-14)
        assert np.all(res["h"][0, 1:] == 0)
        assert M.dequantize_blocks(res["hq"], res["hexp"])[0, 0] == HQ[e]
        assert F.bf16_to_f64(res["row_bits"])[0, :2].tolist() == list(ROWS[e])
    y = [g[0] * ROWS[ids[0]][c] + g[1] * ROWS[ids[1]][c] for c in range(2)]
    assert r["y"][0, :2] == pytest.approx(y, abs=1e-14)
    assert np.all(r["y"][0, 2:] == 0)
    assert F.bf16_to_f64(r["out_bits"])[0, :2].tolist() == list(out01)


def test_hand_worked_with_shared_expert():
    xb, Wr, b, W1, W1s, W2, W2s = _hand_layer([0, 0, 0, 0], shared_expert=True)
    r = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=2, shared=1)
    assert r["ids"][0].tolist() == [3, 1]
    assert r["counts"].tolist() == [0, 1, 0, 1, 1]
    e0, e1 = math.exp(1.5), math.exp(1.0)
    g = [e0 / (e0 + e1), e1 / (e0 + e1)]
    y0 = g[0] * 3.5 + g[1] * -0.5625 + 1.5          # shared row (1.5, 1.5), weight 1
    y1 = g[0] * -1.75 + g[1] * -1.125 + 1.5
    assert r["y"][0, :2] == pytest.approx([y0, y1], abs=1e-14)
    # 3.46624 -> 222/64 ; -0.0140371 -> -230 * 2^-14
    assert F.bf16_to_f64(r["out_bits"])[0, :2].tolist() == [3.46875, -230 * 2.0 ** -14]


def _small_layer(T=24, H=256, Ii=256, E=4, k=2, shared=0, seed=11):
    w = I.Workload("t", T=T, H=H, I=Ii, E=E, k=k, shared=shared, router_std=0.05, bias="uniform")
    x, Wr, b = I.make_routing_inputs(w, seed)
    W1, W1s, W2, W2s = I.make_expert_weights(w, seed)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    return w, xb, Wr.numpy(), b.numpy(), W1.numpy(), W1s.numpy(), W2.numpy(), W2s.numpy()


def test_k_equal_E_reduces_to_dense_weighted_sum():
    w, xb, Wr, b, W1, W1s, W2, W2s = _small_layer(E=4, k=4)
    r = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=4, shared=0)
    s = M.router_scores(xb, Wr)
    full = np.exp(s - s.max(axis=1, keepdims=True))
    full /= full.sum(axis=1, keepdims=True)                    # bias plays no role
    dense = M.dense_reference(xb, Wr, W1, W1s, W2, W2s, full)
    assert np.allclose(r["y"], dense, rtol=1e-12, atol=1e-12)


def test_identical_experts_reduce_to_one_expert():
    w, xb, Wr, b, W1, W1s, W2, W2s = _small_layer(E=4, k=3, shared=0)
    for e in range(1, 4):
        W1[e], W1s[e], W2[e], W2s[e] = W1[0], W1s[0], W2[0], W2s[0]
    r = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=3, shared=0)
    xq, xexp = M.quantize_blocks(F.bf16_to_f64(xb))
    single = M.expert_ffn(xq, xexp, W1[0], W1s[0], W2[0], W2s[0], W1.shape[1] // 2)
    assert np.array_equal(r["out_bits"], single["row_bits"])


def test_output_follows_token_permutation_bitwise():
    w, xb, Wr, b, W1, W1s, W2, W2s = _small_layer(T=30, E=6, k=2, shared=1)
    r = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=2, shared=1)
    pi = np.random.default_rng(0).permutation(30)
    rp = M.forward(xb[pi], Wr, b, W1, W1s, W2, W2s, k=2, shared=1)
    assert np.array_equal(rp["out_bits"], r["out_bits"][pi])


def test_token_subset_matches_full_forward():
    w, xb, Wr, b, W1, W1s, W2, W2s = _small_layer(T=30, E=6, k=2, shared=1)
    r = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=2, shared=1)
    sub = [3, 0, 29, 17]
    rs = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=2, shared=1, tokens=sub)
    assert np.array_equal(rs["out_bits"], r["out_bits"][sub])


def test_doubling_w2_scales_doubles_output_exactly():
    w, xb, Wr, b, W1, W1s, W2, W2s = _small_layer(E=4, k=2, shared=1)
    r = M.forward(xb, Wr, b, W1, W1s, W2, W2s, k=2, shared=1)
    r2 = M.forward(xb, Wr, b, W1, W1s, W2, (W2s + 1).astype(np.uint8), k=2, shared=1)
    assert np.array_equal(r2["y"], 2 * r["y"])
    assert np.array_equal(F.bf16_to_f64(r2["out_bits"]), 2 * F.bf16_to_f64(r["out_bits"]))


def test_activation_quantiser_against_library_codec():
    rng = np.random.default_rng(9)
    x = (rng.normal(0, 1, (16, 512)) * 10.0 ** rng.uniform(-3, 3, (16, 1))).astype(np.float32)
    x[3, :128] = 0.0                                           # all-zero block -> scale 1, codes 0
    xb = x.astype(np.float64)
    codes, p = M.quantize_blocks(xb)
    assert np.all(p[3, 0] == 0) and np.all(codes[3, :128] == 0)
    amax = np.abs(xb.reshape(16, 4, 128)).max(-1)
    assert np.all(amax <= 448 * np.ldexp(1.0, p)) and np.all((amax == 0) | (amax > 224 * np.ldexp(1.0, p)))
    scaled = (xb.reshape(16, 4, 128) / np.ldexp(1.0, p)[..., None]).astype(np.float32)
    ref = scaled.astype(ml_dtypes.float8_e4m3fn).view(np.uint8).reshape(16, 512)
    assert np.array_equal(codes, ref)
    deq = M.dequantize_blocks(codes, p)
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 above the subnormal range
    big = np.abs(scaled.reshape(16, 512)) >= 2.0 ** -6
    assert np.all(np.abs(deq - xb)[big] <= np.abs(xb)[big] * 2.0 ** -4)
