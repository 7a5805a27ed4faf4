"""moe_route_noalloc: routing for callers that cannot allocate device memory.

The entry point keeps its intermediates in a fixed scratch array inside the
library instead of a caller workspace.  Here it is called through the C ABI
twice in a row (different inputs, so the second call must not see the first
call's leftovers) and compared with the plan-based moe_debug_routing on the
same inputs: ids bit for bit, gates within the routing tolerance of the other
GPU tests.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_fp4_moe_b200 import binding
from fp8_fp4_moe_b200 import inputs as I

pytestmark = pytest.mark.gpu

GATE_RTOL, GATE_ATOL = 2e-6, 2e-7


def test_route_noalloc_matches_plan_routing_on_two_calls(cuda_lib):
    w = I.Workload("noalloc", T=333, H=512, I=256, E=64, k=8, shared=1, router_std=0.01, bias="uniform")
    plan = binding.Plan(w.T, w.H, w.I, w.E, w.k, w.shared)
    plan.set_option(binding.MOE_OPT_ROUTER_TC, 0)      # the router kernels the entry point runs
    ids = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    gates = torch.empty(w.T, w.k, dtype=torch.float32, device="cuda")
    for seed in (21, 22):
        x, W_r, bias = (t.cuda() for t in I.make_routing_inputs(w, seed))
        ids.fill_(-1)
        gates.fill_(float("nan"))
        binding.route_noalloc(x, W_r, bias, w.k, topk_ids=ids, gates=gates)
        ref_ids, ref_gates = plan.debug_routing(x, W_r, bias)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids)
        np.testing.assert_allclose(gates.cpu().numpy(), ref_gates.cpu().numpy(), rtol=GATE_RTOL, atol=GATE_ATOL)
        assert torch.all(gates.sum(dim=1).sub(1).abs() < 1e-5)


def test_route_noalloc_rejects_shapes_beyond_its_scratch(cuda_lib):
    L = binding.lib()
    T, H, E, k = 20000, 256, 256, 8            # needs > 16 MiB of scratch
    x = torch.zeros(1, 256, dtype=torch.bfloat16, device="cuda")
    dummy = torch.zeros(16, dtype=torch.float32, device="cuda")
    rc = L.moe_route_noalloc(T, H, E, k, x.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                             dummy.data_ptr(), ctypes.c_void_p(0))
    assert rc == binding.MOE_ERR_WORKSPACE
    assert L.moe_route_noalloc(4, 200, 8, 2, x.data_ptr(), dummy.data_ptr(), dummy.data_ptr(),
                               dummy.data_ptr(), dummy.data_ptr(), None) == binding.MOE_ERR_UNSUPPORTED_SHAPE
