"""Expert-parallel index bookkeeping (fp8_fp4_moe_b200/ep.py) against the single-device oracle.

Host logic only (no GPU).  In one process: a rank's send order is its single-device dispatch
order, grouped by destination; the receive regrouping reproduces the global dispatch order of
every expert.  Over 2 and 4 gloo ranks (torch.distributed.run, 127.0.0.1): token rows travel by
all_to_all_single to their experts' owners and back, and the combined layer output equals the
oracle's single-device forward over all tokens.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest

from fp8_fp4_moe_b200 import ep
from fp8_fp4_moe_b200 import inputs as I
from oracle import moe as M

from parity import bits

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _routing(T=64, E=16, k=4, seed=5):
    w = I.Workload("ep", T=T, H=256, I=256, E=E, k=k, shared=1, router_std=0.05, bias="uniform")
    x, W_r, bias = I.make_routing_inputs(w, seed)
    ids, _, _ = M.route(bits(x), W_r.numpy(), bias.numpy(), k)
    return w, ids


def test_layout_rejects_uneven_sharding():
    with pytest.raises(ValueError):
        ep.EPLayout(E=10, G=4)
    L = ep.EPLayout(E=16, G=4)
    assert L.E_loc == 4 and int(L.owner(13)) == 3 and int(L.local(13)) == 1


@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_send_order_is_the_single_device_dispatch_order(G):
    # one rank holding every token: its send buffer is the oracle's dispatch permutation, and the
    # split sizes are the owners' sums of the per-expert counts
    w, ids = _routing()
    counts, offsets, perm, slot_pos = M.dispatch(ids, w.E, 0)
    sp = ep.send_plan(ids, ep.EPLayout(w.E, G))
    assert np.array_equal(sp.send_copy, perm)
    assert np.array_equal(sp.send_pos, slot_pos)
    assert np.array_equal(sp.expert_counts.reshape(-1), counts[:w.E])
    assert np.array_equal(sp.send_counts, counts[:w.E].reshape(G, -1).sum(axis=1))


@pytest.mark.parametrize("G", [2, 4])
def test_receive_regrouping_matches_the_global_dispatch_of_every_expert(G):
    # ranks hold consecutive token blocks; the receiver's expert-major regrouping of the
    # arrivals (sources in rank order) is the global dispatch order of each of its experts
    w, ids = _routing()
    layout = ep.EPLayout(w.E, G)
    T_r = w.T // G
    counts, offsets, perm, _ = M.dispatch(ids, w.E, 0)
    plans = [ep.send_plan(ids[r * T_r:(r + 1) * T_r], layout) for r in range(G)]
    for d in range(G):
        seg = np.stack([plans[s].expert_counts[d] for s in range(G)])
        rp = ep.recv_plan(seg)
        # arrival buffer of rank d: each source's rows for d, source after source (global copy ids)
        arrivals = []
        for s, sp in enumerate(plans):
            lo = int(sp.send_counts[:d].sum())
            cp = sp.send_copy[lo:lo + int(sp.send_counts[d])]
            arrivals.append((cp // w.k + s * T_r) * w.k + cp % w.k)
        arrivals = np.concatenate(arrivals)
        assert len(arrivals) == int(rp.recv_counts.sum())
        for l in range(layout.E_loc):
            e = d * layout.E_loc + l
            got = arrivals[rp.group_rows[rp.group_offsets[l]:rp.group_offsets[l + 1]]]
            assert np.array_equal(got, perm[offsets[e]:offsets[e + 1]])
            assert rp.group_counts[l] == counts[e]


@pytest.mark.parametrize("G", [2, 4])
def test_expert_parallel_layer_over_gloo_ranks_matches_the_oracle(tmp_path, G):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", str(G),
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join("tests", "ep_worker.py"), str(tmp_path)]
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="", OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-3000:]
    ranks = []
    for i in range(G):
        with open(tmp_path / f"ep_rank{i}.json") as f:
            ranks.append(json.load(f))
    # the single-device oracle over all tokens (same seeded inputs as the worker)
    import torch
    w = I.Workload("ep", T=64, H=256, I=256, E=16, k=4, shared=1, router_std=0.05, bias="uniform")
    x, W_r, bias = I.make_routing_inputs(w, 5)
    W1, W1s, W2, W2s = I.make_expert_weights(w, 5)
    ref = M.forward(x.view(torch.int16).numpy().view(np.uint16), W_r.numpy(), bias.numpy(), W1.numpy(),
                    W1s.numpy(), W2.numpy(), W2s.numpy(), k=w.k, shared=w.shared)
    T_r = w.T // G
    ids = np.concatenate([np.array(d["ids"]) for d in ranks])
    assert np.array_equal(ids, ref["ids"])
    # every expert saw its rows in the single-device dispatch order (global tokens)
    for d in ranks:
        for e, toks in d["order"].items():
            e = int(e)
            want = ref["perm"][ref["offsets"][e]:ref["offsets"][e + 1]] // w.k
            assert toks == want.tolist(), (d["rank"], e)
    # the layer output: float64 y within rounding of the summation order, bf16 outputs equal
    y = np.concatenate([np.array(d["y"]) for d in ranks])
    out = np.concatenate([np.array(d["out_bits"], dtype=np.uint16) for d in ranks])
    assert y.shape == ref["y"].shape
    assert np.max(np.abs(y - ref["y"])) <= 1e-12 * np.max(np.abs(ref["y"]))
    assert np.mean(out != ref["out_bits"]) <= 1e-3
    # rows per rank pair add up to the routed copies
    sent = np.array([d["send_counts"] for d in ranks])
    recv = np.array([d["recv_counts"] for d in ranks])
    assert np.array_equal(sent, recv.T) and int(sent.sum()) == w.T * w.k
    assert all(d["T_r"] == T_r for d in ranks)
