"""Pins for the oracle's router, top-k selection, gates and dispatch.

Selection is checked against brute-force enumeration of every k-subset; gates
against closed forms; dispatch against its defining invariants.
"""
import itertools
import math

import numpy as np
import pytest

from oracle import moe as M
from oracle import screen


def _brute_force_topk(b, k):
    """The unique k-subset whose smallest biased score beats every score left out."""
    E = len(b)
    winners = []
    for S in itertools.combinations(range(E), k):
        rest = [e for e in range(E) if e not in S]
        if not rest or min(b[e] for e in S) > max(b[e] for e in rest):
            winners.append(set(S))
    assert len(winners) == 1
    return winners[0]


@pytest.mark.parametrize("E,k", [(2, 1), (5, 2), (6, 3), (8, 2), (10, 4), (7, 7)])
def test_selection_matches_subset_enumeration(E, k):
    rng = np.random.default_rng(E * 100 + k)
    for _ in range(40):
        s = rng.normal(0, 1, size=(1, E))
        bias = rng.uniform(-0.5, 0.5, size=E).astype(np.float32)
        b = s[0] + bias.astype(np.float64)
        ids = M.select_experts(s, bias, k)[0]
        assert set(ids.tolist()) == _brute_force_topk(b.tolist(), k)
        assert all(b[ids[i]] > b[ids[i + 1]] for i in range(k - 1))      # slot order


def test_combination_count_of_fine_grained_routing():
    # The lesson's fine-grained-experts section counts C(256, 8) ~ 400 trillion
    # expert combinations per token; the enumeration above uses the same count.
    assert math.comb(256, 8) == 409_663_695_276_000
    assert sum(1 for _ in itertools.combinations(range(10), 4)) == math.comb(10, 4)


def test_exact_ties_go_to_lower_id():
    s = np.array([[1.0, 1.0, 0.5, 1.0, 0.25]])
    zero = np.zeros(5, dtype=np.float32)
    assert M.select_experts(s, zero, 2)[0].tolist() == [0, 1]
    assert M.select_experts(s, zero, 3)[0].tolist() == [0, 1, 3]
    # a bias can create the tie: 0.5 + 0.5 == 1.0 exactly
    b = np.array([0, 0, 0.5, 0, 0], dtype=np.float32)
    assert M.select_experts(s, b, 4)[0].tolist() == [0, 1, 2, 3]


def test_bias_moves_selection_but_not_gates():
    s = np.array([[0.5, 1.0, 0.25, 1.5]])
    ids = M.select_experts(s, np.array([0, 0, 1, 0], dtype=np.float32), 2)
    assert ids[0].tolist() == [3, 2]
    g = M.softmax_gates(s, ids)[0]
    e1, e2 = math.exp(1.5), math.exp(0.25)
    assert g[0] == pytest.approx(e1 / (e1 + e2), abs=1e-15)
    assert g[1] == pytest.approx(e2 / (e1 + e2), abs=1e-15)


def test_gates_sum_to_one_and_equal_renormalised_full_softmax():
    rng = np.random.default_rng(3)
    s = rng.normal(0, 2, size=(200, 16))
    bias = rng.uniform(-1, 1, size=16).astype(np.float32)
    for k in (1, 3, 8, 16):
        ids = M.select_experts(s, bias, k)
        g = M.softmax_gates(s, ids)
        assert np.allclose(g.sum(axis=1), 1.0, atol=1e-12, rtol=0)
        full = np.exp(s) / np.exp(s).sum(axis=1, keepdims=True)
        sel = np.take_along_axis(full, ids, axis=1)
        assert np.allclose(g, sel / sel.sum(axis=1, keepdims=True), rtol=1e-12, atol=0)
        if k == 1:
            assert np.all(g == 1.0)


def test_router_scores_are_the_plain_dot_product():
    rng = np.random.default_rng(4)
    import torch
    x = torch.randn(5, 32, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    W = rng.normal(0, 0.1, size=(3, 32)).astype(np.float32)
    s = M.router_scores(xb, W)
    for t in range(5):
        for e in range(3):
            ref = math.fsum(float(x[t, h]) * float(W[e, h]) for h in range(32))
            assert s[t, e] == pytest.approx(ref, rel=1e-14, abs=1e-15)


@pytest.mark.parametrize("T,E,k,shared", [(1, 4, 2, 0), (37, 8, 2, 0), (64, 16, 4, 1), (50, 5, 5, 1)])
def test_dispatch_invariants(T, E, k, shared):
    rng = np.random.default_rng(T + E)
    s = rng.normal(size=(T, E))
    ids = M.select_experts(s, np.zeros(E, np.float32), k)
    counts, offsets, perm, slot_pos = M.dispatch(ids, E, shared)
    R = T * k
    assert counts.sum() == R + shared * T
    assert offsets[0] == 0 and offsets[-1] == R + shared * T and np.all(np.diff(offsets) == counts)
    assert sorted(perm.tolist()) == list(range(R))                  # bijection
    for t in range(T):
        for j in range(k):
            r = slot_pos[t, j]
            assert perm[r] == t * k + j
            e = ids[t, j]
            assert offsets[e] <= r < offsets[e + 1]
    for e in range(E):                                               # ascending tokens
        toks = [perm[r] // k for r in range(offsets[e], offsets[e + 1])]
        assert toks == sorted(toks) and len(set(toks)) == len(toks)
    if shared:
        assert counts[E] == T and offsets[E] == R


def test_margin_screen_detects_close_scores():
    s = np.array([[1.0, 0.9995, 0.5, 0.0], [1.0, 0.9, 0.5, 0.0], [1.0, 0.9, 0.8995, 0.0]])
    ok = screen.margin_ok(s, np.zeros(4, np.float32), 2)
    assert ok.tolist() == [False, True, False]       # third: gap between 2nd and 3rd (k+1-th)
    assert screen.margin_ok(s, np.zeros(4, np.float32), 1).tolist() == [False, True, True]
