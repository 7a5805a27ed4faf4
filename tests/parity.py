"""Shared helpers of the GPU parity tests: build cases, run the oracle, compare."""
from __future__ import annotations

import numpy as np
import torch

from fp8_fp4_moe_b200 import inputs as I
from oracle import formats as F
from oracle import moe as M
from oracle import screen

# Output tolerance of the layer (relative Frobenius, and max-abs relative to rms(out)).
REL_FROB_TOL = 5e-3
MAX_ABS_RMS_TOL = 2e-2
# Gates: fp32 router logits over up to H = 7168 products differ from fp64 by
# ~1e-6..1e-5; a softmax gate's relative error is at most twice the largest
# logit error.
GATE_RTOL, GATE_ATOL = 1e-4, 1e-6
# The requantisation of h (E4M3 code and power-of-two block exponent) is an integer decision
# the kernel takes on its fp32 h, whose value depends on the tensor cores' accumulation order;
# the oracle takes it on the float64 h.  A decision counts as ambiguous when h moved by this
# relative amount (64 fp32 ulps, a few times the spread of fp32 sums over the K of these
# layers; measured flips are about 1 in 10^5 codes) reaches another code or exponent; either
# outcome is then a correct result.
AMBIG_REL = 2.0 ** -18


def bf16_half_ulp(y):
    """Half the bf16 spacing at |y|: the rounding error any bf16 output may carry."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    _, e = np.frexp(np.maximum(a, 2.0 ** -126))     # a in [2^(e-1), 2^e)
    return np.ldexp(1.0, e - 1 - 8)


def bits(x: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> uint16 numpy bit patterns (CPU)."""
    return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def make_case(w: I.Workload, seed: int = 0, screened: bool = True, weight_device="cpu"):
    if screened:
        x, W_r, bias, _ = screen.screened_routing_inputs(w, seed)
    else:
        x, W_r, bias = I.make_routing_inputs(w, seed)
    W1, W1s, W2, W2s = I.make_expert_weights(w, seed, device=weight_device)
    return dict(x=x, W_router=W_r, bias=bias, W1=W1, W1_scales=W1s, W2=W2, W2_scales=W2s)


def to_device(case: dict, device="cuda") -> dict:
    return {k: v.to(device).contiguous() for k, v in case.items()}


_POOL = None
POOL_TIMEOUT_S = 1800


def oracle_pool():
    """Worker processes (spawn start: safe after CUDA is initialised) that evaluate the oracle's
    per-expert FFNs in parallel on the host cores; created on first use, reused by every test.
    A worker that dies breaks the pool with an error instead of leaving a result pending."""
    global _POOL
    if _POOL is None:
        import concurrent.futures as cf
        import multiprocessing as mp
        import os

        from threadpoolctl import threadpool_limits
        n = max(1, min(32, (os.cpu_count() or 2) - 1))
        # one BLAS thread per worker (the workers already use every core between them)
        _POOL = cf.ProcessPoolExecutor(n, mp_context=mp.get_context("spawn"), initializer=threadpool_limits,
                                       initargs=(1,))
    return _POOL


def oracle_forward(case: dict, w: I.Workload, tokens=None, keep_rows=False, parallel=False):
    ffn_map = None
    if parallel:
        pool = oracle_pool()
        ffn_map = lambda f, jobs: pool.map(f, jobs, timeout=POOL_TIMEOUT_S)   # noqa: E731
    return M.forward(bits(case["x"]), case["W_router"].cpu().numpy(), case["bias"].cpu().numpy(),
                     case["W1"].cpu().numpy(), case["W1_scales"].cpu().numpy(), case["W2"].cpu().numpy(),
                     case["W2_scales"].cpu().numpy(), k=w.k, shared=w.shared, tokens=tokens, keep_rows=keep_rows,
                     ffn_map=ffn_map)


def output_errors(gpu_out_bits: np.ndarray, ref_y: np.ndarray):
    got = F.bf16_to_f64(gpu_out_bits)
    diff = got - ref_y
    rms = float(np.sqrt(np.mean(ref_y ** 2)))
    rel_frob = float(np.linalg.norm(diff) / max(np.linalg.norm(ref_y), 1e-300))
    max_abs = float(np.max(np.abs(diff)))
    return rel_frob, max_abs, rms


def h_decision_range(h, hq, hexp):
    """Per element of h [n, I]: the dequantised values [lo, hi] that every correct
    requantisation of h can give, float64 h known up to AMBIG_REL (module note), and the
    oracle's own dequantised value.  lo == hi wherever the decision is unambiguous."""
    h = np.asarray(h, dtype=np.float64)
    n, K = h.shape
    hb = h.reshape(n, K // M.QBLOCK, M.QBLOCK)
    d = AMBIG_REL * np.abs(hb)
    amax = np.abs(hb).max(axis=-1)
    cands = [F.pow2_exponent(amax * (1.0 - AMBIG_REL)), F.pow2_exponent(amax * (1.0 + AMBIG_REL))]
    lo = hi = None
    for p in cands:
        for v in (hb - d, hb + d):
            dq = np.ldexp(F.decode_e4m3(F.encode_e4m3(np.ldexp(v, -p[..., None]))), p[..., None])
            lo = dq if lo is None else np.minimum(lo, dq)
            hi = dq if hi is None else np.maximum(hi, dq)
    own = M.dequantize_blocks(hq, hexp)
    return lo.reshape(n, K), hi.reshape(n, K), own


def decision_slack(case: dict, w: I.Workload, ref: dict) -> np.ndarray:
    """Per output element [tokens, H]: the largest change of the layer output that other
    correct requantisations of h (h_decision_range) can cause, through linear2, the bf16
    rounding of the expert row and the gate.  Zero wherever no decision feeding the element is
    ambiguous.  `ref` from oracle_forward(..., keep_rows=True)."""
    n = len(ref["tokens"])
    slack = np.zeros((n, w.H), dtype=np.float64)
    W2 = case["W2"].cpu().numpy()
    W2s = case["W2_scales"].cpu().numpy()
    gates = ref["gates"][ref["tokens"]]
    for e, (lst, res) in ref["rows"].items():
        lo, hi, own = h_decision_range(res["h"], res["hq"], res["hexp"])
        dev = np.maximum(own - lo, hi - own)
        cols = np.nonzero(dev.any(axis=0))[0]
        if cols.size == 0:
            continue
        # only the weight columns an ambiguous h channel multiplies
        blocks = sorted(set(int(c) // 32 for c in cols))
        wcol = {}
        for b in blocks:
            wb = F.dequant_mxfp4(W2[e][:, b * 16:(b + 1) * 16], W2s[e][:, b:b + 1])   # [H, 32]
            for c in cols[(cols // 32) == b]:
                wcol[int(c)] = np.abs(wb[:, int(c) % 32])
        do = np.zeros((dev.shape[0], w.H), dtype=np.float64)
        for c in cols:
            do += dev[:, c:c + 1] * wcol[int(c)][None, :]
        row = do + np.where(do > 0, 2.0 * bf16_half_ulp(np.abs(res["o"]) + do), 0.0)
        for r, (i, j) in enumerate(lst):
            slack[i] += row[r] * (gates[i, j] if j >= 0 else 1.0)
    return slack


def oracle_forward_with_slack(case: dict, w: I.Workload, tokens=None, parallel=False):
    ref = oracle_forward(case, w, tokens=tokens, keep_rows=True, parallel=parallel)
    return ref, decision_slack(case, w, ref)


def assert_output_close(gpu_out_bits, ref_y, what="", slack=None):
    """Relative Frobenius <= 5e-3 and, per element, |out - y| <= 2e-2 * rms(y) on top of
    the half-ulp the bf16 output format itself may need at that element and of `slack`
    (decision_slack: other correct requantisations of h; zero where there are none).

    y is the oracle's float64 output before its final bf16 rounding.  The
    half-ulp allowance matters only in the tail: at |y| >= 5.12 * rms the bf16
    rounding alone (up to 2^-8 |y|) exceeds 2e-2 * rms, which a full-size
    output (millions of values) reaches even when computed exactly.
    """
    rel_frob, max_abs, rms = output_errors(gpu_out_bits, ref_y)
    got = F.bf16_to_f64(gpu_out_bits)
    assert np.all(np.isfinite(got)), what
    assert rel_frob <= REL_FROB_TOL, f"{what}: rel Frobenius {rel_frob:.3e}"
    base = np.abs(got - ref_y) - bf16_half_ulp(ref_y)
    excess = base if slack is None else base - slack
    worst = int(np.argmax(excess))
    assert excess.flat[worst] <= MAX_ABS_RMS_TOL * rms, (
        f"{what}: |out - y| beyond the bf16 half-ulp {excess.flat[worst]:.3e} > {MAX_ABS_RMS_TOL} * rms "
        f"({rms:.3e}) at y={ref_y.flat[worst]:.5f}, out={got.flat[worst]:.5f}; raw max abs {max_abs:.3e}")
    return rel_frob, max_abs, rms


def slack_needed_fraction(gpu_out_bits, ref_y, slack) -> float:
    """Fraction of output elements that pass the max-abs bound only because of the decision
    slack: beyond 2e-2 * rms(y) + the bf16 half-ulp, within it once the slack is added.  A
    systematic error on near-boundary values would show here; ambiguous decisions alone leave
    it near zero."""
    got = F.bf16_to_f64(gpu_out_bits)
    rms = float(np.sqrt(np.mean(ref_y ** 2)))
    base = np.abs(got - ref_y) - bf16_half_ulp(ref_y)
    return float(np.mean(base > MAX_ABS_RMS_TOL * rms))


def untile_scales(atoms, counts, offsets, bm: int = 128) -> np.ndarray:
    """Per-row UE8M0 codes [rows, K/128] from scale atoms [row tiles, K/128, 512] (uint8).

    Row tile g of expert e = (row tiles of experts before e) + rank // bm (bm = the plan's
    row-tile height, MOE_OPT_TILE_ROWS); the row's code sits at byte (r % 32) * 16 + (r // 32) * 4
    of the atom, r = rank % bm.
    """
    atoms = np.asarray(atoms, dtype=np.uint8)
    counts = np.asarray(counts, dtype=np.int64)
    offsets = np.asarray(offsets, dtype=np.int64)
    mt = (counts + bm - 1) // bm
    mstart = np.concatenate([[0], np.cumsum(mt)])
    rows = int(offsets[-1])
    out = np.zeros((rows, atoms.shape[1]), dtype=np.int64)
    for e in range(len(counts)):
        for rank in range(int(counts[e])):
            g = mstart[e] + rank // bm
            r = rank % bm
            word = atoms[g, :, (r % 32) * 16 + (r // 32) * 4:(r % 32) * 16 + (r // 32) * 4 + 4]
            assert np.all(word == word[:, :1]), "code replicated in all four bytes"
            out[offsets[e] + rank] = word[:, 0]
    return out
