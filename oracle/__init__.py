"""CPU oracle for the FP8 x MXFP4 Mixture-of-Experts layer forward.

TEST INFRASTRUCTURE ONLY.  Only `tests/`, `__graft_entry__.smoke()` and the
CPU-baseline leg of `bench.py` may import anything from this package.  The
CUDA library never links, imports or calls it, and it shares no code, table or
constant generator with the CUDA path: the two meet only at the seeded input
generators in `fp8_fp4_moe_b200/inputs.py`, which hold none of the layer's
arithmetic.

Everything here is plain numpy in float64: exact decoders for E4M3, E2M1, UE8M0
and bf16, a definitional round-to-nearest-even encoder for E4M3 and bf16, and
the layer written stage by stage in the order the pages give it (router ->
biased top-k -> softmax gates -> dispatch -> linear1 -> SwiGLU -> linear2 ->
gate-weighted combine, plus the always-on shared expert).

Parity status: every function is pinned by `tests/test_oracle_*.py` against
something other than itself (library codecs, brute force, closed forms, exact
reductions).  What nothing on the pages can pin -- whether the real DeepGEMM
kernel uses exactly these scaling readings -- is listed as "parity unpinned" in
the design notes; the readings themselves are pinned.
"""
from . import formats, moe  # noqa: F401
