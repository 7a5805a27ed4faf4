"""CUDA path vs the CPU oracle, through the C ABI, on seeded inputs.

Bit-exact: routing ids, dispatch counts/offsets/perm/slot_pos, token-order and
dispatched E4M3 activation codes and scales.  Within tolerance: gates (fp32 vs
fp64 softmax) and layer outputs (relative Frobenius <= 5e-3, max-abs <=
2e-2 * rms(out)).  Sizes span several tiles and ragged tails.
"""
import numpy as np
import pytest
import torch

from fp8_fp4_moe_b200 import binding
from fp8_fp4_moe_b200 import inputs as I
from oracle import formats as F
from oracle import moe as M

from parity import (GATE_ATOL, GATE_RTOL, assert_output_close, bits, h_decision_range, make_case, oracle_forward,
                    oracle_forward_with_slack, to_device, untile_scales)

pytestmark = pytest.mark.gpu


def W(name="t", T=64, H=256, I_=512, E=8, k=2, shared=0, router_std=0.02, bias="zeros"):
    return I.Workload(name, T=T, H=H, I=I_, E=E, k=k, shared=shared, router_std=router_std, bias=bias)


SMALL = {
    "tiny": I.WORKLOADS["tiny"],
    "ragged_shared": W("ragged_shared", T=333, H=384, I_=256, E=16, k=4, shared=1, router_std=0.05, bias="uniform"),
    "t1_k1": W("t1_k1", T=1, H=256, I_=256, E=4, k=1),
    # T <= 16: the GEMMs use the few-token shared-memory layout (16-row A regions, 6 stages)
    "t16_shared": W("t16_shared", T=16, H=512, I_=384, E=4, k=2, shared=1, bias="uniform"),
    "k_eq_E": W("k_eq_E", T=50, H=256, I_=384, E=6, k=6, shared=1),
    "dsv3_like": W("dsv3_like", T=96, H=512, I_=256, E=64, k=8, shared=1, router_std=0.01, bias="uniform"),
    # T >= 64 and E % 16 == 0: tensor-core router; E = 48 leaves most of the 128-expert tile masked
    "tc_router": W("tc_router", T=300, H=1024, I_=256, E=48, k=4, shared=1, router_std=0.02, bias="uniform"),
    # E > 32 with T * E > 16384 and E % 16 != 0: a warp per (token, 2 experts) on CUDA cores (the
    # tiled router would have fewer blocks than SMs)
    "wide_router": W("wide_router", T=500, H=512, I_=256, E=40, k=6, shared=1, router_std=0.02, bias="uniform"),
    # k > 8: the combine keeps up to 16 rows a lane in registers
    "k10": W("k10", T=40, H=256, I_=256, E=24, k=10, shared=1, router_std=0.05, bias="uniform"),
    # H % 224 == 0: linear2 runs 224-row weight tiles with a double-buffered accumulator
    "h896": W("h896", T=200, H=896, I_=256, E=8, k=2, shared=1, bias="uniform"),
    "h1792_t8": W("h1792_t8", T=8, H=1792, I_=256, E=16, k=4, shared=1, router_std=0.01, bias="uniform"),
}


def plan_for(w, swap_rows=None, pair_tiles=None, fused=None, tile_rows=None):
    p = binding.Plan(w.T, w.H, w.I, w.E, w.k, w.shared)
    if tile_rows is not None:
        p.set_option(binding.MOE_OPT_TILE_ROWS, tile_rows)
    if w.H % 224 == 0:
        # these shapes run linear2 on 224-row weight tiles (double-buffered accumulator) at any
        # T; by default only T <= 16 does
        p.set_option(binding.MOE_OPT_L2_TILE_ROWS, 224)
    if swap_rows is not None:
        p.set_option(binding.MOE_OPT_SWAP_ROWS, swap_rows)
    if pair_tiles is not None:
        p.set_option(binding.MOE_OPT_PAIR_TILES, pair_tiles)
    if fused is not None:
        p.set_option(binding.MOE_OPT_FUSED, fused)
    return p


# --------------------------------------------------------------------------- quantisation

@pytest.mark.parametrize("name", ["tiny", "ragged_shared"])
def test_quant_x_bit_exact(cuda_lib, name):
    w = SMALL[name]
    x, _, _ = I.make_routing_inputs(w, 3)
    x = x.clone()
    x[0, :128] = 0.0                               # all-zero block
    x[1, 128:256] = torch.tensor(1e-38).to(torch.bfloat16)   # tiny block -> clamped exponent
    x[2, 5] = -0.0
    x[2, 6] = -1e-30                               # rounds to -0 after scaling
    x[min(3, w.T - 1), 7] = 3.0e38                 # huge value
    p = plan_for(w)
    xq, xs = p.debug_quant_x(x.cuda())
    codes, exps = M.quantize_blocks(F.bf16_to_f64(bits(x)))
    assert np.array_equal(xq.cpu().numpy(), codes)
    assert np.array_equal(xs.cpu().numpy().astype(np.float64), np.ldexp(1.0, exps))


# --------------------------------------------------------------------------- routing

@pytest.mark.parametrize("name", ["tiny", "ragged_shared", "t1_k1", "k_eq_E", "dsv3_like", "tc_router", "wide_router",
                                  "k10"])
def test_routing_bit_exact(cuda_lib, name):
    w = SMALL[name]
    case = make_case(w, seed=5)
    p = plan_for(w)
    d = to_device(case)
    ids, gates = p.debug_routing(d["x"], d["W_router"], d["bias"])
    r_ids, r_gates, _ = M.route(bits(case["x"]), case["W_router"].numpy(), case["bias"].numpy(), w.k)
    assert np.array_equal(ids.cpu().numpy(), r_ids)
    np.testing.assert_allclose(gates.cpu().numpy(), r_gates, rtol=GATE_RTOL, atol=GATE_ATOL)


def test_routing_exact_ties_lower_id(cuda_lib):
    # dyadic router rows: fp32 and fp64 logits are exact and tie exactly
    w = W("ties", T=40, H=256, I_=256, E=8, k=3)
    x = torch.zeros(w.T, w.H, dtype=torch.bfloat16)
    x[:, 0] = 1.0
    x[:, 1] = torch.arange(w.T, dtype=torch.float32).remainder(4).to(torch.bfloat16)
    Wr = torch.zeros(w.E, w.H)
    Wr[:, 0] = torch.tensor([0.5, 0.5, 0.25, 0.5, 0.0, 0.25, 0.5, 0.125])
    Wr[:, 1] = torch.tensor([0.0, 0.0, 0.125, 0.0, 0.25, 0.125, 0.0, 0.0])
    bias = torch.tensor([0, 0, 0, 0, 0, 0, 0.25, 0], dtype=torch.float32)
    p = plan_for(w)
    ids, gates = p.debug_routing(x.cuda(), Wr.cuda(), bias.cuda())
    r_ids, r_gates, _ = M.route(bits(x), Wr.numpy(), bias.numpy(), w.k)
    assert np.array_equal(ids.cpu().numpy(), r_ids)
    np.testing.assert_allclose(gates.cpu().numpy(), r_gates, rtol=1e-6, atol=1e-7)
    assert r_ids[0].tolist() == [6, 0, 1]          # 0.75 > 0.5 == 0.5 (lower id first)


def test_routing_nan_scores_are_never_preferred(cuda_lib):
    # experts 0 and 3 score NaN for every token; tokens 0..4 score NaN everywhere and take the
    # lowest ids (the oracle's stable sort places NaN last); other logits are exact dyadics
    w = W("nan", T=40, H=256, I_=256, E=8, k=3)
    x = torch.zeros(w.T, w.H, dtype=torch.bfloat16)
    x[:, 0] = 1.0
    x[:, 1] = torch.arange(w.T, dtype=torch.float32).remainder(4).to(torch.bfloat16)
    x[:5, 2] = float("nan")
    Wr = torch.zeros(w.E, w.H)
    Wr[:, 0] = torch.tensor([0.0, 0.5, 0.25, 0.0, 0.125, 0.375, 0.0625, 0.75])
    Wr[:, 1] = torch.tensor([0.0, 0.0, 0.125, 0.0, 0.25, 0.0, 0.5, 0.0])
    Wr[:, 2] = 1.0
    Wr[[0, 3], 3] = float("nan")
    bias = torch.zeros(w.E)
    p = plan_for(w)
    ids, gates = p.debug_routing(x.cuda(), Wr.cuda(), bias.cuda())
    r_ids, r_gates, _ = M.route(bits(x), Wr.numpy(), bias.numpy(), w.k)
    ids = ids.cpu().numpy()
    assert np.array_equal(ids, r_ids)
    assert (ids[:5] == [0, 1, 2]).all()
    assert not np.isin(ids[5:], [0, 3]).any()
    np.testing.assert_allclose(gates.cpu().numpy()[5:], r_gates[5:], rtol=1e-6, atol=1e-7)


# --------------------------------------------------------------------------- dispatch

def _ids_case(T, E, k, kind, seed=0):
    rng = np.random.default_rng(seed)
    if kind == "random":
        s = rng.normal(size=(T, E))
    elif kind == "one_expert":      # every token picks expert 0 first (others empty but the top-k)
        s = rng.normal(size=(T, E)) - 10 * np.arange(E)[None, :]
    elif kind == "two_experts":
        s = rng.normal(size=(T, E)) * 1e-3
        s[:, 3] += 100
        s[:, 1] += 50
    else:
        raise ValueError(kind)
    return M.select_experts(s, np.zeros(E, np.float32), k)


@pytest.mark.parametrize("T,E,k,shared,kind", [
    (1, 4, 2, 0, "random"), (33, 8, 2, 1, "random"), (1000, 64, 8, 1, "random"), (4097, 16, 4, 0, "random"),
    (300, 8, 1, 0, "one_expert"), (257, 32, 2, 1, "two_experts"), (64, 5, 5, 0, "random"),
])
def test_dispatch_bit_exact(cuda_lib, T, E, k, shared, kind):
    ids = _ids_case(T, E, k, kind, seed=T)
    w = W("d", T=T, H=256, I_=256, E=E, k=k, shared=shared)
    p = plan_for(w)
    counts, offsets, perm, slot_pos = p.debug_dispatch(torch.from_numpy(ids.astype(np.int32)).cuda())
    rc, rof, rperm, rslot = M.dispatch(ids, E, shared)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), rof)
    assert np.array_equal(perm.cpu().numpy(), rperm)
    assert np.array_equal(slot_pos.cpu().numpy(), rslot)
    assert p.check_status()[0] == 0


def test_dispatch_flags_invalid_ids(cuda_lib):
    w = W("bad", T=40, H=256, I_=256, E=8, k=2)
    p = plan_for(w)
    ids = torch.zeros(w.T, w.k, dtype=torch.int32)
    ids[:, 1] = 1
    ids[7, 1] = 8            # out of range
    ids[9, 1] = 0            # duplicate within a token
    p.debug_dispatch(ids.cuda())
    code, detail = p.check_status()
    assert code == binding.MOE_ERR_DEBUG_BOUNDS and detail[3] in (7, 9)
    assert p.check_status()[0] == 0          # cleared


# --------------------------------------------------------------------------- whole layer

# swap_rows 64: row tiles with <= 64 rows of their expert run transposed (weights as the
# MMA's M side); 0: every tile has 128 token rows
@pytest.mark.parametrize("swap_rows", [64, 0])
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_matches_oracle(cuda_lib, name, swap_rows):
    w = SMALL[name]
    case = make_case(w, seed=7)
    d = to_device(case)
    p = plan_for(w, swap_rows)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    # routing and dispatch inside the forward are bit-exact
    assert np.array_equal(p.region("topk_ids").cpu().numpy(), ref["ids"])
    assert np.array_equal(p.region("counts").cpu().numpy(), ref["counts"])
    assert np.array_equal(p.region("offsets").cpu().numpy(), ref["offsets"])
    assert np.array_equal(p.region("slot_pos").cpu().numpy(), ref["slot_pos"])
    # dispatched activation codes: row slot_pos[t, j] holds token t's codes
    xq = p.region("xq").cpu().numpy()
    xsf = untile_scales(p.region("xsf").cpu().numpy(), ref["counts"], ref["offsets"],
                        p.get_option(binding.MOE_OPT_TILE_ROWS))
    rows = ref["slot_pos"]
    for j in range(w.k):
        assert np.array_equal(xq[rows[:, j]], ref["xq"])
        assert np.array_equal(xsf[rows[:, j]] - 127, ref["xexp"])
    if w.shared:
        R = w.T * w.k
        assert np.array_equal(xq[R:R + w.T], ref["xq"])
    assert_output_close(bits(out), ref["y"], name, slack)


# swap_rows as above; tile_rows 32: row tiles of 32 rows on the 6-stage small-tile layout (the
# default when experts average <= 32 rows), here also on shapes whose experts span several such
# tiles (ragged_shared: ~83 rows per expert, the shared expert 333); 128: the 4-stage layout
# pair_tiles 2: every GEMM on CTA pairs (odd row-tile counts leave the second CTA of a pair
# without rows)
@pytest.mark.parametrize("name,swap_rows,tile_rows,pair_tiles",
                         [("ragged_shared", 64, None, None), ("ragged_shared", 0, 128, None),
                          ("ragged_shared", 0, 32, None), ("dsv3_like", 64, None, None),
                          ("dsv3_like", 0, 32, None), ("dsv3_like", 0, 128, None), ("t16_shared", 0, 32, None),
                          ("h896", 0, None, None), ("h896", 64, None, None), ("h896", 0, 32, None),
                          ("ragged_shared", 0, None, 2), ("wide_router", 0, None, 2), ("h896", 0, None, 2)])
def test_forward_intermediates_match_oracle(cuda_lib, name, swap_rows, tile_rows, pair_tiles):
    w = SMALL[name]
    case = make_case(w, seed=8)
    d = to_device(case)
    p = plan_for(w, swap_rows, tile_rows=tile_rows, pair_tiles=pair_tiles)
    if tile_rows is not None:
        assert p.get_option(binding.MOE_OPT_TILE_ROWS) == tile_rows
    p.forward(**d)
    ref = oracle_forward(case, w, keep_rows=True)
    hq = p.region("hq").cpu().numpy()
    hsf = untile_scales(p.region("hsf").cpu().numpy(), ref["counts"], ref["offsets"],
                        p.get_option(binding.MOE_OPT_TILE_ROWS))
    y = F.bf16_to_f64(bits(p.region("y")))
    offsets = ref["offsets"]
    differ = ambiguous = 0
    for e, (lst, res) in ref["rows"].items():
        # oracle rows for expert e are listed in token order == dispatch order
        rows = np.arange(offsets[e], offsets[e + 1])
        assert len(rows) == len(lst)
        g_h = M.dequantize_blocks(hq[rows], hsf[rows] - 127)
        # every requantised value is one a correct decision gives: the oracle's own, or where h
        # lies on a rounding boundary (within the fp32 accumulation-order spread) its neighbour
        lo, hi, own = h_decision_range(res["h"], res["hq"], res["hexp"])
        assert np.all((g_h >= lo) & (g_h <= hi)), e
        differ += int(np.sum(g_h != own))
        ambiguous += int(np.sum(lo != hi))
        ry = res["o"]
        err = np.linalg.norm(y[rows] - ry) / max(np.linalg.norm(ry), 1e-300)
        assert err < 5e-3, (e, err)
    assert differ <= ambiguous


def test_forward_is_deterministic(cuda_lib):
    w = SMALL["dsv3_like"]
    d = to_device(make_case(w, seed=9, screened=False))
    p = plan_for(w)
    a = p.forward(**d).clone()
    b = p.forward(**d).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("pair_tiles", [0, 2])
def test_forward_all_tokens_on_one_expert(cuda_lib, pair_tiles):
    # the bias forces every token onto expert 2 (many row tiles for one expert, others empty)
    w = W("skew", T=700, H=256, I_=384, E=8, k=1, shared=1)
    case = make_case(w, seed=2, screened=False)
    case["bias"] = torch.tensor([0, 0, 50, 0, 0, 0, 0, 0], dtype=torch.float32)
    d = to_device(case)
    p = plan_for(w, pair_tiles=pair_tiles)
    out = p.forward(**d)
    ref, slack = oracle_forward_with_slack(case, w)
    assert ref["counts"].tolist() == [0, 0, 700, 0, 0, 0, 0, 0, 700]
    assert np.array_equal(p.region("counts").cpu().numpy(), ref["counts"])
    assert_output_close(bits(out), ref["y"], "skew", slack)


def _count_mix_case(counts, H=256, I_=384, seed=3):
    """k = 1 routing with prescribed expert loads: token t carries a +10 spike at channel
    target(t) < E over N(0, 0.1) noise and W_router is the identity on the first E channels,
    so the top-1 logit of token t is expert target(t) by a margin of about 10."""
    E = len(counts)
    target = np.repeat(np.arange(E), counts)
    T = len(target)
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(T, generator=g)
    target = torch.from_numpy(target)[perm]
    w = W("count_mix", T=T, H=H, I_=I_, E=E, k=1, shared=1)
    case = make_case(w, seed=seed, screened=False)
    x = 0.1 * torch.randn(T, H, generator=g)
    x[torch.arange(T), target] += 10.0
    case["x"] = x.to(torch.bfloat16)
    Wr = torch.zeros(E, H)
    Wr[torch.arange(E), torch.arange(E)] = 1.0
    case["W_router"] = Wr
    case["bias"] = torch.zeros(E)
    return w, case


@pytest.mark.parametrize("swap_rows,pair_tiles,fused,H", [(64, 0, 0, 256), (32, 0, 0, 256), (0, 0, 0, 256),
                                                          (0, 2, 0, 256), (0, 0, 1, 256), (64, 0, 1, 256),
                                                          (0, 0, 0, 896), (64, 0, 0, 896), (0, 0, 1, 896),
                                                          (0, 2, 0, 896)])
def test_forward_tile_row_boundaries(cuda_lib, swap_rows, pair_tiles, fused, H):
    # expert loads on both sides of 32, 64, 128 and 256 rows (odd and even row-tile counts for
    # the CTA-pair GEMM), plus an empty expert; H = 896 gives linear2 224-row weight tiles
    counts = [1, 17, 32, 33, 64, 65, 128, 129, 0, 200, 256, 257, 384]
    w, case = _count_mix_case(counts, H=H)
    d = to_device(case)
    p = plan_for(w, swap_rows, pair_tiles, fused)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    assert ref["counts"].tolist() == counts + [w.T]
    assert np.array_equal(p.region("counts").cpu().numpy(), ref["counts"])
    assert_output_close(bits(out), ref["y"],
                        f"count_mix H={H} swap_rows={swap_rows} pair_tiles={pair_tiles} fused={fused}", slack)


# CTA-pair GEMMs forced on the small shapes (auto mode uses them from 256 rows per expert on)
@pytest.mark.parametrize("name", ["tiny", "ragged_shared", "k_eq_E", "tc_router"])
def test_forward_pair_tiles_match_oracle(cuda_lib, name):
    w = SMALL[name]
    case = make_case(w, seed=11)
    d = to_device(case)
    p = plan_for(w, pair_tiles=2)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    assert_output_close(bits(out), ref["y"], name + " pairs", slack)
    # the single-CTA kernel forms the same products; only the fp32 summation may differ
    p1 = plan_for(w, pair_tiles=0)
    out1 = p1.forward(**d)
    a = F.bf16_to_f64(bits(out))
    b = F.bf16_to_f64(bits(out1))
    assert np.linalg.norm(a - b) <= 1e-3 * np.linalg.norm(b)


# every step in one persistent cooperative kernel: each router variant (tensor cores for
# ragged_shared / dsv3_like / tc_router, a warp per (expert, K part) over all tokens for t1_k1 /
# t16_shared / h1792_t8, block per expert and token for tiny / k_eq_E / k10 / h896, warp per
# token and 2 experts for wide_router), routing and dispatch bit-exact, outputs in tolerance
@pytest.mark.parametrize("name", list(SMALL))
def test_forward_fused_matches_oracle(cuda_lib, name):
    w = SMALL[name]
    case = make_case(w, seed=13)
    d = to_device(case)
    p = plan_for(w, fused=1)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    assert np.array_equal(p.region("topk_ids").cpu().numpy(), ref["ids"])
    assert np.array_equal(p.region("counts").cpu().numpy(), ref["counts"])
    assert np.array_equal(p.region("offsets").cpu().numpy(), ref["offsets"])
    assert np.array_equal(p.region("slot_pos").cpu().numpy(), ref["slot_pos"])
    np.testing.assert_allclose(p.region("gates").cpu().numpy(), ref["gates"], rtol=GATE_RTOL, atol=GATE_ATOL)
    assert_output_close(bits(out), ref["y"], name + " fused", slack)
    # repeated launches reuse the grid barrier words
    out2 = p.forward(**d).clone()
    assert p.check_status()[0] == 0
    assert torch.equal(out2.view(torch.int16), out.view(torch.int16))


def test_fused_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    w = SMALL["tiny"]
    case = make_case(w, seed=1)
    d = to_device(case)
    p = plan_for(w, fused=1)
    p.set_option(binding.MOE_OPT_TIMEOUT_NS, 50_000_000)      # 50 ms
    p.set_option(binding.MOE_OPT_INJECT_FAULT, 1)             # one stage of linear1 never arrives
    p.forward(**d)
    code, _ = p.check_status()
    assert code == binding.MOE_ERR_DEVICE_TIMEOUT
    p.set_option(binding.MOE_OPT_INJECT_FAULT, 0)
    p.set_option(binding.MOE_OPT_TIMEOUT_NS, 2_000_000_000)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    assert_output_close(bits(out), ref["y"], "fused after timeout", slack)


def test_update_bias_matches_oracle_and_evens_out_loads(cuda_lib):
    # one step is bit-exact against the oracle's rule on the forward's counts; a loop of
    # forward + update brings a skewed router's loads close to uniform
    w = W("bias_loop", T=100, H=256, I_=256, E=8, k=2)
    case = make_case(w, seed=21, screened=False)
    Wr = case["W_router"].clone()
    Wr[:, 0] += torch.linspace(0.6, -0.6, w.E)
    case["W_router"] = Wr
    x = case["x"].clone()
    x[:, 0] = 1.0
    case["x"] = x
    d = to_device(case)
    p = plan_for(w)
    bias = torch.zeros(w.E, device="cuda")
    d["bias"] = bias
    p.forward(**d)
    counts = p.region("counts").cpu().numpy()[: w.E]
    before = bias.cpu().numpy().copy()
    p.update_bias(bias, 0.02)
    assert np.array_equal(bias.cpu().numpy(), M.update_bias(before, counts, w.T, w.k, 0.02))
    start = counts.max() / (w.T * w.k / w.E)
    ratios = []
    for _ in range(50):
        p.forward(**d)
        p.update_bias(bias, 0.02)
        ratios.append(p.region("counts").cpu().numpy()[: w.E].max() / (w.T * w.k / w.E))
    assert p.check_status()[0] == 0
    assert start > 2.0
    assert min(ratios[-10:]) < 1.3


def test_token_permutation_permutes_output(cuda_lib):
    w = SMALL["ragged_shared"]
    case = make_case(w, seed=4, screened=False)
    d = to_device(case)
    p = plan_for(w)
    a = p.forward(**d).clone()
    pi = torch.randperm(w.T, generator=torch.Generator().manual_seed(0))
    d2 = dict(d)
    d2["x"] = d["x"][pi.cuda()].contiguous()
    b = p.forward(**d2)
    assert torch.equal(b.view(torch.int16), a[pi.cuda()].view(torch.int16))


def test_doubling_w2_scales_doubles_output(cuda_lib):
    w = SMALL["tiny"]
    d = to_device(make_case(w, seed=6, screened=False))
    p = plan_for(w)
    a = p.forward(**d).clone().float()
    d["W2_scales"] = d["W2_scales"] + 1
    b = p.forward(**d).float()
    assert torch.equal(b, 2 * a)


def test_static_weights_reuse_prepared_scales(cuda_lib):
    w = SMALL["ragged_shared"]
    case = make_case(w, seed=12, screened=False)
    d = to_device(case)
    p = plan_for(w)
    ref = p.forward(**d).clone()
    p.set_option(binding.MOE_OPT_STATIC_WEIGHTS, 1)
    p.prepare_weights(d["W1_scales"], d["W2_scales"])
    a = p.forward(**d).clone()
    assert torch.equal(a.view(torch.int16), ref.view(torch.int16))
    # in-place change of the scales is only seen after an explicit prepare
    d["W2_scales"].add_(1)
    stale = p.forward(**d).clone()
    assert torch.equal(stale.view(torch.int16), ref.view(torch.int16))
    p.prepare_weights(d["W1_scales"], d["W2_scales"])
    b = p.forward(**d).float()
    assert torch.equal(b, 2 * ref.float())
    p.set_option(binding.MOE_OPT_STATIC_WEIGHTS, 0)
    c = p.forward(**d).float()
    assert torch.equal(c, b)


def test_graph_replay_matches_direct_launches(cuda_lib):
    w = SMALL["dsv3_like"]
    d = to_device(make_case(w, seed=13, screened=False))
    p = plan_for(w)
    ref = p.forward(**d).clone()
    p.set_option(binding.MOE_OPT_GRAPH, 1)
    out = torch.empty_like(ref)
    for _ in range(3):                                  # record, then replay
        out.zero_()
        p.forward(**d, out=out)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    # a replay reads the current contents of the same buffers
    x2 = make_case(w, seed=14, screened=False)["x"].cuda()
    d["x"].copy_(x2)
    p.forward(**d, out=out)
    p.set_option(binding.MOE_OPT_GRAPH, 0)
    ref2 = p.forward(**d).clone()
    assert torch.equal(out.view(torch.int16), ref2.view(torch.int16))
    assert p.check_status()[0] == 0


@pytest.mark.parametrize("name", ["t16_shared", "dsv3_like", "tc_router", "ragged_shared", "h1792_t8"])
def test_dependent_launch_matches_plain_stream_order(cuda_lib, name):
    # kernels that start early and wait on the device give the same bits as plain stream order,
    # with and without a recorded graph, with the weight scales re-laid out in the middle of
    # every forward (the default) and with that step skipped (static weights)
    w = SMALL[name]
    d = to_device(make_case(w, seed=21, screened=False))
    p = plan_for(w)
    p.set_option(binding.MOE_OPT_DEPENDENT_LAUNCH, 0)
    ref = p.forward(**d).clone()
    p.set_option(binding.MOE_OPT_DEPENDENT_LAUNCH, 1)
    for graph in (0, 1):
        p.set_option(binding.MOE_OPT_GRAPH, graph)
        for _ in range(3):
            out = p.forward(**d)
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), graph
    p.set_option(binding.MOE_OPT_GRAPH, 0)
    p.set_option(binding.MOE_OPT_STATIC_WEIGHTS, 1)
    for _ in range(2):
        out = p.forward(**d)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert p.check_status()[0] == 0


@pytest.mark.parametrize("name", ["t1_k1", "t16_shared", "h1792_t8"])
def test_chained_gemms_match_two_launches_bitwise(cuda_lib, name):
    # linear1 and linear2 in one cooperative launch with per-expert counters compute the same
    # products in the same order as two launches: the same bits, graph or not (h1792_t8 runs
    # linear2 on 224-row tiles, the others on 256-row tiles)
    w = SMALL[name]
    case = make_case(w, seed=23, screened=False)
    d = to_device(case)
    p = plan_for(w)
    ref = p.forward(**d).clone()
    p.set_option(binding.MOE_OPT_CHAIN, 1)
    for graph in (0, 1):
        p.set_option(binding.MOE_OPT_GRAPH, graph)
        for _ in range(3):
            out = p.forward(**d)
            assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), graph
    assert p.check_status()[0] == 0
    ref_o, slack = oracle_forward_with_slack(case, w)
    assert_output_close(bits(out), ref_o["y"], name + " chained", slack)


def test_chained_gemms_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    # one linear1 stage never fills: that CTA's MMA wait runs out, its expert's counter never
    # completes, and every linear2 producer waiting on it runs out too -- all bounded
    w = SMALL["t16_shared"]
    case = make_case(w, seed=1)
    d = to_device(case)
    p = plan_for(w)
    p.set_option(binding.MOE_OPT_CHAIN, 1)
    p.set_option(binding.MOE_OPT_TIMEOUT_NS, 50_000_000)
    p.set_option(binding.MOE_OPT_INJECT_FAULT, 1)
    p.forward(**d)
    code, detail = p.check_status()
    assert code == binding.MOE_ERR_DEVICE_TIMEOUT
    assert detail[1] & 0xF00 in (0x100, 0x200, 0x300, 0x400, 0xA00)
    p.set_option(binding.MOE_OPT_INJECT_FAULT, 0)
    p.set_option(binding.MOE_OPT_TIMEOUT_NS, 2_000_000_000)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    assert_output_close(bits(out), ref["y"], "chained after timeout", slack)


# --------------------------------------------------------------------------- failure detection

def test_bounded_wait_reports_timeout_and_context_survives(cuda_lib):
    w = SMALL["tiny"]
    case = make_case(w, seed=1)
    d = to_device(case)
    p = plan_for(w)
    p.set_option(binding.MOE_OPT_TIMEOUT_NS, 50_000_000)      # 50 ms
    p.set_option(binding.MOE_OPT_INJECT_FAULT, 1)             # scale factors of one stage never arrive
    p.forward(**d)
    code, detail = p.check_status()
    assert code == binding.MOE_ERR_DEVICE_TIMEOUT
    assert detail[1] & 0xF00 in (0x300, 0x400, 0x100, 0x200)
    p.set_option(binding.MOE_OPT_INJECT_FAULT, 0)
    p.set_option(binding.MOE_OPT_TIMEOUT_NS, 2_000_000_000)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    assert_output_close(bits(out), ref["y"], "after timeout", slack)


# zero padding of the A rows a 128-row tile does not fill changes no result: the padded rows only
# reach accumulator rows that are never stored
@pytest.mark.parametrize("name", ["ragged_shared", "dsv3_like", "h896"])
def test_zero_padding_changes_no_bit(cuda_lib, name):
    w = SMALL[name]
    d = to_device(make_case(w, seed=31, screened=False))
    outs = []
    for zero_pad in (2, 1):                       # never, always
        p = plan_for(w, tile_rows=128)
        p.set_option(binding.MOE_OPT_ZERO_PAD, zero_pad)
        assert p.get_option(binding.MOE_OPT_ZERO_PAD) == zero_pad
        outs.append(p.forward(**d).clone())
        assert p.check_status()[0] == 0
        outs.append(p.region("y").clone())
    assert torch.equal(outs[0].view(torch.int16), outs[2].view(torch.int16))
    assert torch.equal(outs[1].view(torch.int16), outs[3].view(torch.int16))


# A grid of a few CTAs (MOE_OPT_MAX_SMS) gives every CTA many tiles and every epilogue warp many
# scatter and combine batches (the fused kernel's per-warp mbarrier phases wrap many times): the
# arithmetic of a tile or an item does not depend on which CTA runs it, so the output equals the
# full grid's bit for bit, and the oracle's within tolerance.
@pytest.mark.parametrize("name,fused,pair_tiles", [("ragged_shared", 1, None), ("k10", 1, None), ("h896", 1, None),
                                                   ("ragged_shared", 0, None), ("tc_router", 0, 2)])
def test_few_ctas_match_the_full_grid(cuda_lib, name, fused, pair_tiles):
    w = SMALL[name]
    case = make_case(w, seed=41)
    d = to_device(case)
    outs = []
    for max_sms in (0, 2, 7):
        p = plan_for(w, fused=fused, pair_tiles=pair_tiles)
        p.set_option(binding.MOE_OPT_MAX_SMS, max_sms)
        outs.append(p.forward(**d).clone())
        assert p.check_status()[0] == 0, max_sms
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    ref, slack = oracle_forward_with_slack(case, w)
    assert_output_close(bits(outs[1]), ref["y"], f"{name} fused={fused} on 2 CTAs", slack)


# Enough (token, 256-channel slice) items (T * slices >= 32768) for the many-token scatters: the
# scatter kernel's four slices per warp, and the single kernel's eight quantised slices staged in
# shared memory and sent to each dispatched row with one bulk copy.  The dispatched codes and
# scale bytes are the oracle's bit for bit, with one group of slices per token (H = 2048) and with
# a ragged last group ending in half a slice (H = 2176)
@pytest.mark.parametrize("fused", [0, 1])
@pytest.mark.parametrize("H", [2048, 2176])
def test_bulk_scatter_matches_oracle(cuda_lib, H, fused):
    w = W(f"bulk_scatter_{H}", T=4096, H=H, I_=256, E=16, k=4, shared=1, router_std=0.05, bias="uniform")
    case = make_case(w, seed=43)
    d = to_device(case)
    p = plan_for(w, fused=fused)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    ref, slack = oracle_forward_with_slack(case, w)
    assert np.array_equal(p.region("topk_ids").cpu().numpy(), ref["ids"])
    assert np.array_equal(p.region("offsets").cpu().numpy(), ref["offsets"])
    assert np.array_equal(p.region("slot_pos").cpu().numpy(), ref["slot_pos"])
    assert np.array_equal(p.region("perm").cpu().numpy()[:w.T * w.k], ref["perm"])
    xq = p.region("xq").cpu().numpy()
    xsf = untile_scales(p.region("xsf").cpu().numpy(), ref["counts"], ref["offsets"],
                        p.get_option(binding.MOE_OPT_TILE_ROWS))
    rows = ref["slot_pos"]
    for j in range(w.k):
        assert np.array_equal(xq[rows[:, j]], ref["xq"])
        assert np.array_equal(xsf[rows[:, j]] - 127, ref["xexp"])
    R = w.T * w.k
    assert np.array_equal(xq[R:R + w.T], ref["xq"])
    assert np.array_equal(xsf[R:R + w.T] - 127, ref["xexp"])
    assert_output_close(bits(out), ref["y"], w.name, slack)
