"""Pins of the oracle's dense FP8 x FP4 GEMM (operand formats of "DeepSeek Mega MoE /
DeepGEMM mega kernel", "TL;DR"): a hand-worked product, element-by-element brute force from
the format definitions, and exact scale doublings."""
import numpy as np

from oracle import moe as M

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _e4m3(code):
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 7
    return s * (m / 8.0 * 2.0 ** -6 if e == 0 else (1 + m / 8.0) * 2.0 ** (e - 7))


def _e2m1(nib):
    return (-1.0 if nib & 8 else 1.0) * E2M1[nib & 7]


def test_hand_worked_single_product():
    K, N = 128, 128
    a = np.zeros((1, K), np.uint8)
    a[0, 3] = 0x3C                                   # E4M3 1.5
    a_s = np.full((1, 1), 128, np.uint8)             # x2
    b = np.zeros((N, K // 2), np.uint8)
    b[5, 1] = 0x50                                   # element 3 = high nibble of byte 1 = E2M1 3.0
    b_s = np.full((N, K // 32), 127, np.uint8)
    b_s[5, 0] = 126                                  # x0.5 on the block holding element 3
    out, bits = M.dense_gemm(a, a_s, b, b_s)
    exp = np.zeros((1, N))
    exp[0, 5] = 1.5 * 2 * 3.0 * 0.5
    assert np.array_equal(out, exp)
    assert bits[0, 5] == 0x4090                      # bf16 4.5


def _random_case(rng, Mr, N, K):
    a = rng.integers(0, 256, (Mr, K)).astype(np.uint8)
    a[(a & 0x7F) == 0x7F] = 0x3C                     # no NaN codes
    a_s = rng.integers(118, 136, (Mr, K // 128)).astype(np.uint8)
    b = rng.integers(0, 256, (N, K // 2)).astype(np.uint8)
    b_s = rng.integers(120, 132, (N, K // 32)).astype(np.uint8)
    return a, a_s, b, b_s


def test_brute_force_from_format_definitions():
    rng = np.random.default_rng(5)
    Mr, N, K = 3, 128, 256
    a, a_s, b, b_s = _random_case(rng, Mr, N, K)
    out, _ = M.dense_gemm(a, a_s, b, b_s)
    for m in range(Mr):
        for n in (0, 1, 17, 127):
            acc = 0.0
            for k in range(K):
                av = _e4m3(int(a[m, k])) * 2.0 ** (int(a_s[m, k // 128]) - 127)
                byte = int(b[n, k // 2])
                nib = byte & 0xF if k % 2 == 0 else byte >> 4   # low nibble = even element
                bv = _e2m1(nib) * 2.0 ** (int(b_s[n, k // 32]) - 127)
                acc += av * bv
            assert abs(out[m, n] - acc) <= 1e-12 * max(1.0, abs(acc)), (m, n)


def test_scale_increments_double_a_row_and_a_column_exactly():
    rng = np.random.default_rng(6)
    a, a_s, b, b_s = _random_case(rng, 4, 128, 256)
    out, _ = M.dense_gemm(a, a_s, b, b_s)
    a_s2 = a_s.copy()
    a_s2[2] += 1
    out2, _ = M.dense_gemm(a, a_s2, b, b_s)
    assert np.array_equal(out2[2], 2 * out[2])
    assert np.array_equal(np.delete(out2, 2, 0), np.delete(out, 2, 0))
    b_s2 = b_s.copy()
    b_s2[7] += 1
    out3, _ = M.dense_gemm(a, a_s, b, b_s2)
    assert np.array_equal(out3[:, 7], 2 * out[:, 7])
    assert np.array_equal(np.delete(out3, 7, 1), np.delete(out, 7, 1))
