"""Dense FP8 x FP4 GEMM (moe_gemm_fp8_fp4) against the oracle on seeded operands: shapes with
ragged row tiles, a partial 256-row weight tile and several K blocks; bf16 outputs within the
layer's output tolerance."""
import numpy as np
import pytest
import torch

from fp8_fp4_moe_b200 import binding
from oracle import moe as M

from parity import assert_output_close, bits

pytestmark = pytest.mark.gpu


def _operands(seed, Mr, N, K):
    rng = np.random.default_rng(seed)
    a = rng.integers(0, 256, (Mr, K)).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] = 0x3C                     # no NaN codes
    a_s = rng.integers(118, 136, (Mr, K // 128)).astype(np.uint8)
    b = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    b_s = rng.integers(120, 132, (N, K // 32)).astype(np.uint8)
    return a, a_s, b, b_s


@pytest.mark.parametrize("Mr,N,K", [(1, 128, 128), (77, 384, 256), (300, 256, 512), (129, 1024, 1024),
                                    (513, 640, 384)])
def test_dense_gemm_matches_oracle(cuda_lib, Mr, N, K):
    a, a_s, b, b_s = _operands(Mr * 7 + N + K, Mr, N, K)
    dev = [torch.from_numpy(t).cuda() for t in (a, a_s, b, b_s)]
    out, ws = binding.gemm_fp8_fp4(*dev)
    torch.cuda.synchronize()
    assert ws[:4].view(torch.int32).item() == 0
    ref, _ = M.dense_gemm(a, a_s, b, b_s)
    assert_output_close(bits(out), ref, f"dense {Mr}x{N}x{K}")


def test_dense_gemm_row_and_column_scale_doubling(cuda_lib):
    a, a_s, b, b_s = _operands(3, 200, 256, 256)
    out = binding.gemm_fp8_fp4(*[torch.from_numpy(t).cuda() for t in (a, a_s, b, b_s)])[0]
    a_s[5] += 1
    b_s[9] += 1
    out2 = binding.gemm_fp8_fp4(*[torch.from_numpy(t).cuda() for t in (a, a_s, b, b_s)])[0]
    o, o2 = out.float(), out2.float()
    assert torch.equal(o2[5, :9], 2 * o[5, :9]) and torch.equal(o2[5, 10:], 2 * o[5, 10:])
    assert torch.equal(o2[:5, 9], 2 * o[:5, 9]) and torch.equal(o2[6:, 9], 2 * o[6:, 9])
    assert torch.equal(o2[5, 9], 4 * o[5, 9])
