"""Seeded synthetic workloads for the FP8 x MXFP4 MoE layer.

This module only DRAWS inputs.  It holds none of the layer's arithmetic: no
routing, no activation quantisation, no GEMM.  The one piece of number-format
code here is the fixture quantiser that turns N(0, std) expert weights into
MXFP4 bytes (E2M1 codes + one UE8M0 scale per 32 along K); the layer only ever
*decodes* that format, so both the CUDA path and the CPU oracle consume the very
same bytes and this choice can never affect parity.

Workload shapes follow the configurations the pages' benchmark is quoted on
(DeepGEMM "Mega MoE" PR #316 batch points of 1/512/8192/32768 tokens per rank,
plus a Mixtral-shaped layer and a tiny layer); value distributions are the ones
stated with each configuration.

Conventions (all tensors row-major, contiguous):
  x          bf16  [T, H]
  W_router   fp32  [E, H]          routed experts only
  bias       fp32  [E]             selection-only bias
  W1         uint8 [E+s, 2I, H/2]  rows 0..I-1 gate, I..2I-1 up; byte j packs
                                   element 2j (low nibble) and 2j+1 (high nibble)
  W1_scales  uint8 [E+s, 2I, H/32] UE8M0, one per 32 consecutive K elements
  W2         uint8 [E+s, H, I/2]
  W2_scales  uint8 [E+s, H, I/32]
Expert index E (the last one) is the shared expert when shared == 1.
"""
from __future__ import annotations

import dataclasses

import torch

__all__ = ["Workload", "WORKLOADS", "make_routing_inputs", "make_expert_weights",
           "make_inputs", "redraw_token_row", "ZIPF_BETA_T8192"]

# Zipf(s=1.1) offset strength for the skewed-prefill workload.  Written by
# oracle/calibrate_zipf.py (seed 0): the busiest expert then receives ~10x the
# mean load.  See that script for the bisection.
ZIPF_BETA_T8192 = 0.25


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    k: int
    shared: int
    router_std: float
    bias: str            # "zeros" | "uniform" | "zipf"
    weight_std: float = 0.02
    description: str = ""

    @property
    def n_experts_total(self) -> int:
        return self.E + self.shared

    @property
    def routed_rows(self) -> int:
        return self.T * self.k

    @property
    def total_rows(self) -> int:
        return self.T * self.k + self.shared * self.T

    def flops(self) -> float:
        """Effective FLOPs of one layer forward: 6*H*I per (token, expert) pair."""
        return 6.0 * self.H * self.I * (self.k + self.shared) * self.T

    def expert_weight_bytes(self) -> int:
        """MXFP4 bytes of one expert (W1 + W2, codes + scales)."""
        return 3 * self.H * self.I // 2 + 3 * self.H * self.I // 32

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T, name=f"{self.name}@T{T}")

    def with_experts(self, E: int) -> "Workload":
        return dataclasses.replace(self, E=E, k=min(self.k, E), name=f"{self.name}@E{E}")


WORKLOADS = {
    "tiny": Workload("tiny", T=64, H=256, I=512, E=8, k=2, shared=0, router_std=0.02,
                     bias="zeros", description="tiny MoE layer T=64 H=256 I=512 E=8 k=2"),
    "mixtral": Workload("mixtral", T=4096, H=4096, I=14336, E=8, k=2, shared=0,
                        router_std=0.02, bias="zeros",
                        description="Mixtral-shaped layer T=4096 H=4096 I=14336 E=8 k=2"),
    "dsv3_t1": Workload("dsv3_t1", T=1, H=7168, I=2048, E=256, k=8, shared=1,
                        router_std=0.01, bias="uniform",
                        description="DeepSeek-V3-shaped decode T=1 H=7168 I=2048 E=256+1 k=8"),
    "dsv3_t512": Workload("dsv3_t512", T=512, H=7168, I=2048, E=256, k=8, shared=1,
                          router_std=0.01, bias="uniform",
                          description="DeepSeek-V3-shaped decode T=512 H=7168 I=2048 E=256+1 k=8"),
    "dsv3_t8192_zipf": Workload("dsv3_t8192_zipf", T=8192, H=7168, I=2048, E=256, k=8,
                                shared=1, router_std=0.01, bias="zipf",
                                description="DeepSeek-V3-shaped prefill T=8192, Zipf(1.1)-skewed routing"),
    "dsv3_t32768": Workload("dsv3_t32768", T=32768, H=7168, I=2048, E=256, k=8, shared=1,
                            router_std=0.01, bias="zeros",
                            description="large-batch prefill T=32768 H=7168 I=2048 E=256+1 k=8"),
}


def _gen(seed: int, *stream: int, device="cpu") -> torch.Generator:
    """An independent generator per (seed, tensor id, ...) tuple."""
    h = seed & 0xFFFFFFFF
    for s in stream:
        h = (h * 1_000_003 + (s & 0xFFFFFFFF) + 0x9E3779B9) & 0xFFFFFFFFFFFF
    g = torch.Generator(device=device)
    g.manual_seed(h)
    return g


def zipf_offsets(E: int, beta: float, s: float = 1.1) -> torch.Tensor:
    """Per-expert Zipf(s) logit offset, rank r = e + 1, zero mean over experts."""
    r = torch.arange(1, E + 1, dtype=torch.float64)
    lg = s * torch.log(r)
    return (beta * (-lg + lg.mean())).to(torch.float32)


def make_routing_inputs(w: Workload, seed: int = 0, zipf_beta: float | None = None):
    """x (bf16 [T,H]), W_router (fp32 [E,H]) and bias (fp32 [E]) on the CPU.

    Always drawn on the CPU so that the token/router values are identical on
    every machine, whichever device the expert weights are drawn on.
    """
    x = torch.randn(w.T, w.H, generator=_gen(seed, 1), dtype=torch.float32).to(torch.bfloat16)
    W_r = torch.randn(w.E, w.H, generator=_gen(seed, 2), dtype=torch.float32) * w.router_std
    if w.bias == "zeros":
        bias = torch.zeros(w.E, dtype=torch.float32)
    elif w.bias == "uniform":
        bias = (torch.rand(w.E, generator=_gen(seed, 3), dtype=torch.float32) * 0.1 - 0.05)
    elif w.bias == "zipf":
        bias = zipf_offsets(w.E, ZIPF_BETA_T8192 if zipf_beta is None else zipf_beta)
    else:
        raise ValueError(w.bias)
    return x, W_r.contiguous(), bias.contiguous()


def redraw_token_row(seed: int, t: int, attempt: int, H: int) -> torch.Tensor:
    """A fresh bf16 N(0,1) row for token t (used when a token fails the margin screen)."""
    return torch.randn(H, generator=_gen(seed, 7, t, attempt), dtype=torch.float32).to(torch.bfloat16)


# --- fixture MXFP4 quantiser (weights only; never on the layer's path) --------------

_E2M1_GRID = (0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def _mxfp4_quantise(w: torch.Tensor):
    """w fp32 [rows, K] -> (packed uint8 [rows, K/2], UE8M0 uint8 [rows, K/32]).

    Per 32-block: smallest integer p with amax <= 6 * 2^p (p = 0 for an all-zero
    block); codes = nearest point of the E2M1 grid to w / 2^p, ties to the even
    code.
    """
    rows, K = w.shape
    assert K % 32 == 0
    blk = w.view(rows, K // 32, 32)
    amax = blk.abs().amax(dim=-1)
    m, e = torch.frexp(amax)                      # amax = m * 2^e, m in [0.5, 1)
    p = torch.where(m <= 0.75, e - 3, e - 2)
    p = torch.where(amax == 0, torch.zeros_like(p), p).clamp(-127, 127)
    v = blk / torch.pow(2.0, p.to(torch.float32)).unsqueeze(-1)
    grid = torch.tensor(_E2M1_GRID, dtype=torch.float32, device=w.device)
    a = v.abs().clamp(max=6.0)
    hi = torch.searchsorted(grid, a.contiguous()).clamp(max=7)
    lo = (hi - 1).clamp(min=0)
    dlo = a - grid[lo]
    dhi = grid[hi] - a
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (hi % 2 == 0))
    idx = torch.where(pick_hi, hi, lo)
    idx = torch.where(a == grid[lo], lo, idx)
    code = idx | (torch.signbit(v) & (idx != 0)).to(idx.dtype) << 3
    code = code.to(torch.uint8).view(rows, K)
    packed = code[:, 0::2] | (code[:, 1::2] << 4)
    scales = (p + 127).to(torch.uint8)
    return packed.contiguous(), scales.contiguous()


def make_expert_weights(w: Workload, seed: int = 0, device="cpu", experts=None):
    """MXFP4 expert weights, drawn N(0, weight_std) per expert and quantised.

    Returns W1, W1_scales, W2, W2_scales (uint8 tensors on `device`).
    `experts` optionally restricts the draw to a list of expert ids (the other
    experts are left zero) -- used by CPU timing samples.
    """
    n = w.n_experts_total
    W1 = torch.zeros(n, 2 * w.I, w.H // 2, dtype=torch.uint8, device=device)
    W1s = torch.zeros(n, 2 * w.I, w.H // 32, dtype=torch.uint8, device=device)
    W2 = torch.zeros(n, w.H, w.I // 2, dtype=torch.uint8, device=device)
    W2s = torch.zeros(n, w.H, w.I // 32, dtype=torch.uint8, device=device)
    ids = range(n) if experts is None else experts
    dev = torch.device(device)
    for e in ids:
        g1 = _gen(seed, 100, e, 1, device=dev.type)
        g2 = _gen(seed, 100, e, 2, device=dev.type)
        w1 = torch.randn(2 * w.I, w.H, generator=g1, device=dev, dtype=torch.float32) * w.weight_std
        W1[e], W1s[e] = _mxfp4_quantise(w1)
        del w1
        w2 = torch.randn(w.H, w.I, generator=g2, device=dev, dtype=torch.float32) * w.weight_std
        W2[e], W2s[e] = _mxfp4_quantise(w2)
        del w2
    return W1, W1s, W2, W2s


def make_inputs(w: Workload, seed: int = 0, device="cpu"):
    """All layer inputs as a dict of torch tensors (routing inputs moved to `device`)."""
    x, W_r, bias = make_routing_inputs(w, seed)
    W1, W1s, W2, W2s = make_expert_weights(w, seed, device)
    return dict(x=x.to(device), W_router=W_r.to(device), bias=bias.to(device),
                W1=W1, W1_scales=W1s, W2=W2, W2_scales=W2s)


def mxfp4_bytes(w: Workload) -> int:
    return w.n_experts_total * w.expert_weight_bytes()


def describe(w: Workload) -> str:
    return (f"{w.name}: T={w.T} H={w.H} I={w.I} E={w.E}+{w.shared} k={w.k} "
            f"flops={w.flops() / 1e12:.3f}T weights={mxfp4_bytes(w) / 1e9:.2f}GB")


if __name__ == "__main__":  # pragma: no cover
    for w in WORKLOADS.values():
        print(describe(w))
