"""moe_route_noalloc: routing for callers that cannot allocate device memory.

Some callers cannot call cudaMalloc (or torch's allocator) at the moment they need a routing
decision: a serving loop that runs inside a fixed, pre-carved memory pool, allocator hooks that
must not re-enter an allocator, runtimes that only hand over raw buffers and a stream.  This
entry point keeps its intermediates in a fixed scratch array inside the library instead of a
caller workspace.

Each case calls it through the C ABI twice in a row (different inputs, so the second call must
not see the first call's leftovers in the shared scratch array) and compares it with the
plan-based moe_debug_routing on the same inputs (ids bit for bit, gates within 2e-6) and with the
oracle on margin-screened inputs (ids bit for bit, gates within the routing tolerance of the other
GPU tests).  The shapes reach every router kernel the entry point can pick.  This file is collected
last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from fp8_fp4_moe_b200 import binding
from fp8_fp4_moe_b200 import inputs as I
from oracle import moe as M
from oracle import screen

from parity import GATE_ATOL, GATE_RTOL, bits

pytestmark = pytest.mark.gpu

SAME_KERNEL_RTOL, SAME_KERNEL_ATOL = 2e-6, 2e-7

# one shape per router kernel of the entry point
CASES = {
    "smem_router": dict(T=64, H=256, E=8, k=2),        # E <= 8, T >= 64: W_router staged in shared memory
    "split_router": dict(T=4, H=512, E=16, k=4),       # T * E <= 4096: block per (expert, token)
    "warp8_router": dict(T=200, H=384, E=32, k=6),     # E <= 32: warp per (token, 8 experts)
    "warp2_router": dict(T=100, H=512, E=64, k=8),     # T * E <= 16384: warp per (token, 2 experts)
    "warp2_few_tiles": dict(T=333, H=512, E=64, k=8),  # T * E > 16384, but 6 router tiles: warp kernel
    "tiled_router": dict(T=2400, H=256, E=256, k=8),   # >= 148 tiles of 64 x 64: the tiled router
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_route_noalloc_matches_plan_routing_and_oracle_on_two_calls(cuda_lib, name):
    c = CASES[name]
    w = I.Workload(name, T=c["T"], H=c["H"], I=256, E=c["E"], k=c["k"], shared=0, router_std=0.02,
                   bias="uniform")
    plan = binding.Plan(w.T, w.H, w.I, w.E, w.k, w.shared)
    plan.set_option(binding.MOE_OPT_ROUTER_TC, 0)      # the router kernels the entry point runs
    ids = torch.empty(w.T, w.k, dtype=torch.int32, device="cuda")
    gates = torch.empty(w.T, w.k, dtype=torch.float32, device="cuda")
    for seed in (21, 22):
        x, W_r, bias, _ = screen.screened_routing_inputs(w, seed)
        xd, Wd, bd = x.cuda(), W_r.cuda(), bias.cuda()
        ids.fill_(-1)
        gates.fill_(float("nan"))
        binding.route_noalloc(xd, Wd, bd, w.k, topk_ids=ids, gates=gates)
        ref_ids, ref_gates = plan.debug_routing(xd, Wd, bd)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids)
        np.testing.assert_allclose(gates.cpu().numpy(), ref_gates.cpu().numpy(), rtol=SAME_KERNEL_RTOL,
                                   atol=SAME_KERNEL_ATOL)
        o_ids, o_gates, _ = M.route(bits(x), W_r.numpy(), bias.numpy(), w.k)
        assert np.array_equal(ids.cpu().numpy(), o_ids)
        np.testing.assert_allclose(gates.cpu().numpy(), o_gates, rtol=GATE_RTOL, atol=GATE_ATOL)


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


def test_route_noalloc_rejects_buffers_not_on_the_current_device(cuda_lib):
    """Host buffers are not device memory of the current device: rejected before any launch."""
    L = binding.lib()
    T, H, E, k = 4, 256, 8, 2
    xh = torch.zeros(T, H, dtype=torch.bfloat16)
    wh = torch.zeros(E, H, dtype=torch.float32)
    bh = torch.zeros(E, dtype=torch.float32)
    ih = torch.zeros(T, k, dtype=torch.int32)
    gh = torch.zeros(T, k, dtype=torch.float32)
    xd, wd, bd = xh.cuda(), wh.cuda(), bh.cuda()
    idd, gd = ih.cuda(), gh.cuda()
    for args in ((xh, wd, bd, idd, gd), (xd, wh, bd, idd, gd), (xd, wd, bh, idd, gd), (xd, wd, bd, ih, gd),
                 (xd, wd, bd, idd, gh)):
        rc = L.moe_route_noalloc(T, H, E, k, *(t.data_ptr() for t in args), None)
        assert rc == binding.MOE_ERR_INVALID_ARG
    torch.cuda.synchronize()
