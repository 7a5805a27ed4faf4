"""Parity at the full workload sizes, in the launch configuration the benchmark times.

The layer runs on every token; the oracle recomputes routing and dispatch for all tokens (bit-exact
comparison) and the expert FFN + combine for a stratified subset of tokens (each output row depends
only on its own token, so the subset is exact).  The subset reaches the places where a tile-count
bug would hide:
  * the last dispatched row of every expert that has rows (the ragged end of its last row tile);
  * one row in every STRIDE-th row tile of every expert (every row tile of the busiest expert of
    the Zipf-skewed layer: its ~20 row tiles are the long tail of that launch);
  * a few uniformly drawn tokens.
Besides the layer output, the sampled dispatched rows of the expert-row buffer (linear2's bf16
output, before the combine) are compared with the oracle's per-expert rows.  Inputs pass the
top-k margin screen.  The oracle's expert FFNs run in a process pool on the host cores.
"""
import numpy as np
import pytest
import torch

from fp8_fp4_moe_b200 import binding
from fp8_fp4_moe_b200 import inputs as I
from oracle import formats as F

from parity import (GATE_ATOL, GATE_RTOL, assert_output_close, bits, make_case, oracle_forward_with_slack,
                    slack_needed_fraction)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

# uniformly drawn tokens on top of the stratified rows, and the row-tile stride
RANDOM_TOKENS = {"mixtral": 8, "dsv3_t1": 1, "dsv3_t512": 8, "dsv3_t8192_zipf": 8, "dsv3_t32768": 8}
TILE_STRIDE = {"mixtral": 16, "dsv3_t1": 1, "dsv3_t512": 1, "dsv3_t8192_zipf": 16, "dsv3_t32768": 16}
# bound on the output elements that need the decision slack to pass (see slack_needed_fraction)
SLACK_NEEDED_MAX = 1e-3
# expert rows (bf16 linear2 output) against the oracle's, relative Frobenius per expert
ROW_REL_TOL = 5e-3
# separate launches and the single persistent kernel for every workload; the chained
# linear1 -> linear2 launch for single-token decode
CASES = [(n, 0, 0) for n in RANDOM_TOKENS] + [(n, 1, 0) for n in RANDOM_TOKENS] + [("dsv3_t1", 0, 1)]


def stratified_rows(counts, offsets, stride, busiest, rng):
    """Dispatched rows to check: the last row of every expert with rows, and one random row in
    every `stride`-th row tile of each expert (every row tile of expert `busiest`)."""
    rows = set()
    for e in range(len(counts)):
        c = int(counts[e])
        if c == 0:
            continue
        o = int(offsets[e])
        rows.add(o + c - 1)
        n_tiles = (c + 127) // 128
        st = 1 if e == busiest else stride
        for g in range(0, n_tiles, st):
            lo, hi = g * 128, min(c, (g + 1) * 128)
            rows.add(o + int(rng.integers(lo, hi)))
    return np.array(sorted(rows), dtype=np.int64)


def row_tokens(rows, perm, T, k):
    """Token of each dispatched row: perm entry t*k + j for routed rows, row R + t for shared."""
    R = T * k
    return np.where(rows < R, perm[np.minimum(rows, R - 1)] // k, rows - R)


@pytest.mark.parametrize("name,fused,chain", CASES)
def test_full_size_stratified_parity(cuda_lib, name, fused, chain):
    w = I.WORKLOADS[name]
    case = make_case(w, seed=0, screened=True, weight_device="cuda")
    d = {k: v.cuda().contiguous() for k, v in case.items()}
    p = binding.Plan(w.T, w.H, w.I, w.E, w.k, w.shared)
    p.set_option(binding.MOE_OPT_FUSED, fused)
    p.set_option(binding.MOE_OPT_CHAIN, chain)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    counts = p.region("counts").cpu().numpy()
    offsets = p.region("offsets").cpu().numpy()
    perm = p.region("perm").cpu().numpy()
    rng = np.random.default_rng(1)
    busiest = int(np.argmax(counts[:w.E])) if name == "dsv3_t8192_zipf" else -1
    rows = stratified_rows(counts, offsets, TILE_STRIDE[name], busiest, rng)
    tokens = np.unique(np.concatenate([row_tokens(rows, perm, w.T, w.k),
                                       rng.choice(w.T, size=min(RANDOM_TOKENS[name], w.T), replace=False)]))
    ref, slack = oracle_forward_with_slack(case, w, tokens=tokens, parallel=True)
    # routing and dispatch of every token, bit for bit
    assert np.array_equal(p.region("topk_ids").cpu().numpy(), ref["ids"])
    assert np.array_equal(counts, ref["counts"])
    assert np.array_equal(offsets, ref["offsets"])
    assert np.array_equal(perm, ref["perm"])
    assert np.array_equal(p.region("slot_pos").cpu().numpy(), ref["slot_pos"])
    np.testing.assert_allclose(p.region("gates").cpu().numpy(), ref["gates"], rtol=GATE_RTOL, atol=GATE_ATOL)
    # the layer output of the sampled tokens
    got = bits(out)[tokens]
    assert_output_close(got, ref["y"], name, slack)
    frac = slack_needed_fraction(got, ref["y"], slack)
    assert frac <= SLACK_NEEDED_MAX, f"{name}: {frac:.2e} of the outputs pass only with the decision slack"
    # the sampled tokens' dispatched rows of the expert-row buffer, expert by expert
    y_rows = p.region("y")
    pos = {int(t): i for i, t in enumerate(tokens)}
    R = w.T * w.k
    for e, (lst, res) in ref["rows"].items():
        want_rows = []
        for i, j in lst:
            t = int(tokens[i])
            want_rows.append(int(ref["slot_pos"][t, j]) if j >= 0 else R + t)
        got_rows = F.bf16_to_f64(bits(y_rows[torch.as_tensor(want_rows, device=y_rows.device)]))
        ry = res["o"]
        err = np.linalg.norm(got_rows - ry) / max(np.linalg.norm(ry), 1e-300)
        assert err < ROW_REL_TOL, (name, e, err)
    # every stratified row was compared (its token is in the sample)
    assert all(int(t) in pos for t in row_tokens(rows, perm, w.T, w.k))
    assert torch.isfinite(out.float()).all()
    del p, d, out, y_rows
    torch.cuda.empty_cache()
