"""The MoE layer forward, written stage by stage in float64 (test infrastructure only).

Sources (page title, section):
  [MoE]   "전문가 혼합(Mixture of Experts; MoE)" lesson -- sections "FFN 교체",
          "부하 분산 문제", "공유 전문가", "Step 1: 라우터", "Step 2: 100개 토큰 라우팅하기".
  [Mega]  "Mega MoE" wiki -- sections "한 줄 정의", "어떻게 작동하나".
  [DG]    "DeepSeek Mega MoE / DeepGEMM mega kernel" -- "TL;DR", "Thông số kỹ thuật".
  [Play]  "Mixture-of-Experts 플레이북" -- section "작동 방식".

Readings where the pages are silent (each listed in the design notes):
  * scores are the raw router logits x . W_r (no softmax/sigmoid before
    selection); bias is added for selection only;
  * ties in the biased score go to the lower expert id; slots are ordered by
    descending biased score;
  * no routed scaling factor; the shared expert has weight 1;
  * SwiGLU is silu(gate) * up with W1 rows 0..I-1 = gate, I..2I-1 = up;
  * activations are quantised per token per 128 channels to E4M3 with a
    power-of-two scale (smallest 2^p with amax <= 448 * 2^p, p >= -126, p = 0
    for an all-zero block); the same rule requantises the SwiGLU output;
  * each expert's output row is rounded to bf16 before the combine; the combine
    sums in slot order, then adds the shared row, and rounds to bf16 once;
  * dispatch order: expert-major, ascending token id inside an expert, shared
    expert rows last in token order.
"""
from __future__ import annotations

import numpy as np

from . import formats as F

QBLOCK = 128   # activation quantisation block (channels)


# ----------------------------------------------------------------------------- routing

def router_scores(x_bits, W_router) -> np.ndarray:
    """s[t, e] = sum_h x[t, h] * W_r[e, h] in float64.

    [MoE] "FFN 교체": the router is one linear layer producing (N_tokens, E)
    scores; "Step 1: 라우터": each score is the dot product of the hidden vector
    with that expert's router row.  [Play] "작동 방식" step 1.
    """
    x = F.bf16_to_f64(x_bits)
    W = np.asarray(W_router, dtype=np.float32).astype(np.float64)
    return x @ W.T


def select_experts(scores, bias, k: int) -> np.ndarray:
    """Top-k expert ids per token by descending (score + bias), lower id first on ties.

    [MoE] "Step 1: 라우터": the biased scores are sorted in descending order with
    a stable sort and the first k indices kept; "부하 분산 문제" item 3: the
    per-expert bias only steers selection.
    """
    s = np.asarray(scores, dtype=np.float64)
    b = np.asarray(bias, dtype=np.float32).astype(np.float64)
    biased = s + b[None, :]
    order = np.argsort(-biased, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def softmax_gates(scores, ids) -> np.ndarray:
    """Softmax over the UNBIASED scores of the selected experts, max subtracted.

    [MoE] "Step 1: 라우터": gates come from the original scores of the chosen
    experts, never from the biased ones.
    """
    chosen = np.take_along_axis(np.asarray(scores, dtype=np.float64), ids, axis=1)
    m = chosen.max(axis=1, keepdims=True)
    ex = np.exp(chosen - m)
    return ex / ex.sum(axis=1, keepdims=True)


def route(x_bits, W_router, bias, k: int):
    s = router_scores(x_bits, W_router)
    ids = select_experts(s, bias, k)
    return ids, softmax_gates(s, ids), s


# ----------------------------------------------------------------------------- dispatch

def dispatch(ids, n_routed: int, shared: int):
    """Canonical in-memory dispatch of token copies to experts.

    [Mega] "한 줄 정의"/"어떻게 작동하나": dispatch sends each token to its
    experts.  On one device this is a permutation of the T*k token copies into
    expert-major order; inside an expert the copies are in ascending token
    order.  With a shared expert ([MoE] "공유 전문가": every token passes it),
    rows R..R+T-1 hold token t at row R + t.

    Returns counts [E+s], offsets [E+s+1], perm [R] (entry t*k + j at the row
    that token t's j-th copy occupies) and slot_pos [T, k] (that row).
    """
    ids = np.asarray(ids, dtype=np.int64)
    T, k = ids.shape
    n_tot = n_routed + shared
    counts = np.zeros(n_tot, dtype=np.int64)
    for e in range(n_routed):
        counts[e] = np.count_nonzero(ids == e)
    if shared:
        counts[n_routed] = T
    offsets = np.zeros(n_tot + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    R = T * k
    perm = np.empty(R, dtype=np.int64)
    slot_pos = np.empty((T, k), dtype=np.int64)
    fill = offsets[:n_routed].copy()
    for t in range(T):                      # ascending token order
        for j in range(k):
            e = ids[t, j]
            slot_pos[t, j] = fill[e]
            perm[fill[e]] = t * k + j
            fill[e] += 1
    return counts, offsets, perm, slot_pos


# ----------------------------------------------------------------------------- quantisation

def quantize_blocks(values, block: int = QBLOCK):
    """Per-row, per-`block`-channel E4M3 quantisation with power-of-two scales.

    Returns (codes uint8 [n, K], exps int64 [n, K/block]); value ~ decode(code) * 2^exp.
    The division by 2^p is exact, so the only rounding is the E4M3 one.
    """
    v = np.asarray(values, dtype=np.float64)
    n, K = v.shape
    assert K % block == 0
    blk = v.reshape(n, K // block, block)
    amax = np.abs(blk).max(axis=-1)
    p = F.pow2_exponent(amax)
    scaled = np.ldexp(blk, -p[..., None])
    codes = F.encode_e4m3(scaled).reshape(n, K)
    return codes, p


def dequantize_blocks(codes, exps, block: int = QBLOCK) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    n, K = c.shape
    vals = F.decode_e4m3(c).reshape(n, K // block, block)
    return np.ldexp(vals, np.asarray(exps)[..., None]).reshape(n, K)


# ----------------------------------------------------------------------------- experts

def silu(z):
    """silu(z) = z * sigmoid(z) = z / (1 + exp(-z))."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def expert_ffn(xq, xexp, W1_e, W1s_e, W2_e, W2s_e, I: int):
    """One expert on its rows: linear1 -> SwiGLU -> E4M3 requant -> linear2 -> bf16.

    [DG] "TL;DR": linear1 (FP8 x FP4) -> SwiGLU -> linear2 (FP8 x FP4);
    [MoE] "FFN 교체": each expert is a SwiGLU-family FFN.

    xq/xexp: the rows' E4M3 codes [n, H] and exponents [n, H/128].
    Returns dict(a, h, hq, hexp, o, row_bits).
    """
    xd = dequantize_blocks(xq, xexp)                      # exact
    W1 = F.dequant_mxfp4(W1_e, W1s_e)                     # [2I, H] exact
    a = xd @ W1.T                                         # [n, 2I]
    h = silu(a[:, :I]) * a[:, I:]
    hq, hexp = quantize_blocks(h)
    hd = dequantize_blocks(hq, hexp)
    W2 = F.dequant_mxfp4(W2_e, W2s_e)                     # [H, I] exact
    o = hd @ W2.T                                         # [n, H]
    return dict(a=a, h=h, hq=hq, hexp=hexp, o=o, row_bits=F.f64_to_bf16(o))


# ----------------------------------------------------------------------------- forward

def _expert_job(job):
    """expert_ffn on one expert's rows; `job` = its argument tuple (a picklable unit of work)."""
    return expert_ffn(*job)


def forward(x_bits, W_router, bias, W1, W1_scales, W2, W2_scales, k: int, shared: int,
            tokens=None, keep_rows: bool = False, ffn_map=None):
    """The whole layer for all tokens, or only for `tokens` (routing is always global).

    [MoE] "FFN 교체": y = sum over the top-k experts of gate * Expert_e(x);
    [Play] "작동 방식" step 3 (weighted sum) and the shared expert every token
    passes.  Each output row depends only on its own token, so computing a
    subset of tokens is exact.

    `ffn_map` (default: the builtin map) evaluates the experts' FFNs, which are
    independent of one another: a process pool's map gives the same numbers.

    Returns a dict with ids, gates, scores, counts, offsets, perm, slot_pos,
    the token-order x quantisation (xq, xexp), out_bits [n_tok, H] (bf16 bits),
    y [n_tok, H] (float64 before the final rounding) and `tokens`.
    """
    x_bits = np.asarray(x_bits, dtype=np.uint16)
    T, H = x_bits.shape
    W1 = np.asarray(W1)
    E = np.asarray(W_router).shape[0]
    n_tot = E + shared
    I = W1.shape[1] // 2
    assert W1.shape == (n_tot, 2 * I, H // 2)

    ids, gates, scores = route(x_bits, W_router, bias, k)
    counts, offsets, perm, slot_pos = dispatch(ids, E, shared)
    R = T * k

    tok = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    x = F.bf16_to_f64(x_bits[tok])
    xq, xexp = quantize_blocks(x)                         # per token, before dispatch

    # rows needed: (token index in `tok`, slot j or -1 for shared) grouped per expert
    rows_by_expert = {e: [] for e in range(n_tot)}
    for i, t in enumerate(tok):
        for j in range(k):
            rows_by_expert[int(ids[t, j])].append((i, j))
        if shared:
            rows_by_expert[E].append((i, -1))

    n = len(tok)
    row_vals = np.zeros((n, k + shared, H), dtype=np.float64)   # bf16 rows as float64
    extras = {}
    used = [e for e in range(n_tot) if rows_by_expert[e]]
    sels = {e: np.array([i for i, _ in rows_by_expert[e]], dtype=np.int64) for e in used}
    jobs = ((xq[sels[e]], xexp[sels[e]], W1[e], W1_scales[e], W2[e], W2_scales[e], I) for e in used)
    for e, res in zip(used, (map if ffn_map is None else ffn_map)(_expert_job, jobs)):
        lst = rows_by_expert[e]
        rv = F.bf16_to_f64(res["row_bits"])
        for r, (i, j) in enumerate(lst):
            row_vals[i, j if j >= 0 else k] = rv[r]
        if keep_rows:
            extras[e] = (lst, res)

    y = np.zeros((n, H), dtype=np.float64)
    for j in range(k):                                    # slot order, then shared
        y = y + gates[tok, j][:, None] * row_vals[:, j]
    if shared:
        y = y + row_vals[:, k]
    out_bits = F.f64_to_bf16(y)
    return dict(ids=ids, gates=gates, scores=scores, counts=counts, offsets=offsets,
                perm=perm, slot_pos=slot_pos, R=R, xq=xq, xexp=xexp, tokens=tok,
                out_bits=out_bits, y=y, rows=extras)


def dense_reference(x_bits, W_router, W1, W1_scales, W2, W2_scales, gates_full):
    """Gate-weighted sum over ALL routed experts with given per-token gates [T, E].

    Used only to pin forward() in the k = E case, where top-k selection keeps
    every expert and the combine must reduce to this dense sum.
    """
    x = F.bf16_to_f64(np.asarray(x_bits, dtype=np.uint16))
    xq, xexp = quantize_blocks(x)
    E = gates_full.shape[1]
    I = np.asarray(W1).shape[1] // 2
    y = np.zeros_like(x)
    for e in range(E):
        res = expert_ffn(xq, xexp, W1[e], W1_scales[e], W2[e], W2_scales[e], I)
        y = y + gates_full[:, e][:, None] * F.bf16_to_f64(res["row_bits"])
    return y


# ----------------------------------------------------------------------------- bias update

def update_bias(bias, counts, T: int, k: int, gamma: float) -> np.ndarray:
    """One auxiliary-loss-free balancing step on the per-expert selection bias.

    [MoE] "부하 분산 문제" item 3 and "Step 2: 100개 토큰 라우팅하기": after a step,
    every expert used more than its target share loses gamma, every expert used
    less gains gamma.  Readings: the target is the mean load T*k/E (compared
    exactly as the integers T*k and count*E); an expert exactly at the target
    keeps its bias; bias is fp32 (the layer's bias input) and each update is one
    fp32 addition.  `counts` are the E routed experts' loads.
    """
    b = np.asarray(bias, dtype=np.float32)
    c = np.asarray(counts, dtype=np.int64)
    E = b.shape[0]
    diff = np.int64(T) * k - c * E                      # > 0: under-used, < 0: over-used
    step = np.where(diff > 0, np.float32(gamma), np.where(diff < 0, -np.float32(gamma), np.float32(0)))
    return (b + step.astype(np.float32)).astype(np.float32)


# ----------------------------------------------------------------------------- dense GEMM

def dense_gemm(a_codes, a_scale_codes, b_packed, b_scale_codes):
    """out[m, n] = sum_k deq(A)[m, k] * deq(B)[n, k] in float64, and its bf16 rounding.

    [DG] "TL;DR": the FP8 x FP4 product of the expert FFN, here for one dense operand pair.
    A: E4M3 codes [M, K] with UE8M0 codes [M, K/128] (one power of two per row per 128
    channels, the layer's activation format); B: packed E2M1 [N, K/2] with UE8M0 codes
    [N, K/32].  Returns (out_f64 [M, N], out_bf16_bits [M, N]).
    """
    a_exp = np.asarray(a_scale_codes, dtype=np.int64) - 127
    a = dequantize_blocks(np.asarray(a_codes, dtype=np.uint8), a_exp)
    b = F.dequant_mxfp4(np.asarray(b_packed, dtype=np.uint8), np.asarray(b_scale_codes, dtype=np.uint8))
    out = a @ b.T
    return out, F.f64_to_bf16(out)
