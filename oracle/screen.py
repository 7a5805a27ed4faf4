"""Top-k margin screen for parity inputs (test infrastructure only).

Routing ids are compared bit for bit between the CUDA path (fp32 logits) and
this oracle (fp64 logits).  That comparison is only meaningful when no two of a
token's top k+1 biased scores are closer than the arithmetic difference of the
two sides, so parity inputs are screened: a token passes when every gap between
consecutive entries of its k+1 largest biased fp64 scores is at least `margin`
(1e-3); a failing token's x row is redrawn from its own sub-seeded stream until
it passes.  With the gaps that large both the selected set and the slot order
are fixed.
"""
from __future__ import annotations

import numpy as np
import torch

from fp8_fp4_moe_b200 import inputs as _inputs

from . import moe as _moe

MARGIN = 1e-3


def margin_ok(scores, bias, k: int, margin: float = MARGIN) -> np.ndarray:
    """bool [T]: True where the top k+1 biased scores are pairwise >= margin apart."""
    b = np.asarray(scores, dtype=np.float64) + np.asarray(bias, dtype=np.float32).astype(np.float64)[None, :]
    E = b.shape[1]
    top = -np.sort(-b, axis=1)[:, :min(k + 1, E)]
    if top.shape[1] < 2:
        return np.ones(b.shape[0], dtype=bool)
    gaps = top[:, :-1] - top[:, 1:]
    return np.all(gaps >= margin, axis=1)


def screened_routing_inputs(w, seed: int = 0, margin: float = MARGIN, max_attempts: int = 1000):
    """Routing inputs of workload `w` with every token passing the margin screen.

    Returns (x bf16 [T,H], W_router, bias, n_redrawn) as CPU torch tensors.
    """
    x, W_r, bias = _inputs.make_routing_inputs(w, seed)
    xb = x.view(torch.int16).numpy().view(np.uint16)
    s = _moe.router_scores(xb, W_r.numpy())
    ok = margin_ok(s, bias.numpy(), w.k, margin)
    redrawn = 0
    for t in np.nonzero(~ok)[0]:
        for attempt in range(max_attempts):
            row = _inputs.redraw_token_row(seed, int(t), attempt, w.H)
            rb = row.view(torch.int16).numpy().view(np.uint16)
            st = _moe.router_scores(rb[None, :], W_r.numpy())
            if margin_ok(st, bias.numpy(), w.k, margin)[0]:
                x[t] = row
                redrawn += 1
                break
        else:
            raise RuntimeError(f"token {t}: no row passed the margin screen")
    return x, W_r, bias, redrawn
