"""Parity at the full workload sizes, in the launch configuration the benchmark times.

The layer runs on every token; the oracle recomputes routing and dispatch for
all tokens (bit-exact comparison) and the expert FFN + combine for a sampled
subset of tokens (each output row depends only on its own token, so the subset
is exact).  Inputs pass the top-k margin screen.
"""
import numpy as np
import pytest
import torch

from fp8_fp4_moe_b200 import binding
from fp8_fp4_moe_b200 import inputs as I

from parity import GATE_ATOL, GATE_RTOL, assert_output_close, bits, make_case, oracle_forward_with_slack

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

SAMPLES = {"mixtral": 24, "dsv3_t1": 1, "dsv3_t512": 8, "dsv3_t8192_zipf": 8, "dsv3_t32768": 6}
# separate launches for every workload; the single persistent kernel for three of them; the
# chained linear1 -> linear2 launch for single-token decode
CASES = [(n, 0, 0) for n in SAMPLES] + [("dsv3_t1", 1, 0), ("dsv3_t512", 1, 0), ("mixtral", 1, 0),
                                        ("dsv3_t1", 0, 1)]


@pytest.mark.parametrize("name,fused,chain", CASES)
def test_full_size_sampled_parity(cuda_lib, name, fused, chain):
    w = I.WORKLOADS[name]
    case = make_case(w, seed=0, screened=True, weight_device="cuda")
    d = {k: v.cuda().contiguous() for k, v in case.items()}
    p = binding.Plan(w.T, w.H, w.I, w.E, w.k, w.shared)
    p.set_option(binding.MOE_OPT_FUSED, fused)
    p.set_option(binding.MOE_OPT_CHAIN, chain)
    out = p.forward(**d)
    assert p.check_status()[0] == 0
    rng = np.random.default_rng(1)
    tokens = np.sort(rng.choice(w.T, size=min(SAMPLES[name], w.T), replace=False))
    if name == "dsv3_t8192_zipf":
        # include a token of the busiest expert
        ids = p.region("topk_ids").cpu().numpy()
        busiest = np.bincount(ids.ravel(), minlength=w.E).argmax()
        tokens = np.unique(np.append(tokens, np.nonzero((ids == busiest).any(axis=1))[0][0]))
    ref, slack = oracle_forward_with_slack(case, w, tokens=tokens)
    assert np.array_equal(p.region("topk_ids").cpu().numpy(), ref["ids"])
    assert np.array_equal(p.region("counts").cpu().numpy(), ref["counts"])
    assert np.array_equal(p.region("offsets").cpu().numpy(), ref["offsets"])
    assert np.array_equal(p.region("slot_pos").cpu().numpy(), ref["slot_pos"])
    np.testing.assert_allclose(p.region("gates").cpu().numpy(), ref["gates"], rtol=GATE_RTOL, atol=GATE_ATOL)
    got = bits(out)[tokens]
    assert_output_close(got, ref["y"], name, slack)
    assert torch.isfinite(out.float()).all()
    del p, d, out
    torch.cuda.empty_cache()
