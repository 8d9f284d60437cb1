"""Pins for the oracle GEMM on dequantised MX operands.

Exact rational brute force on tiny shapes (the operands are dyadic, so the FP64
result must be exact when partial sums stay within 53 bits), the alpha / bias /
row-subset plumbing, and the error-quadrature property printed on the ork-driver
W4A4 page (weight-only and activation-only errors add in quadrature).
"""

import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from conftest import golden
from mxfp4_block_scaled_mxq_b200 import inputs

E2M1 = {int(c, 16): Fraction(v) for c, v in golden("e2m1_values.txt")}


def _random_mx(rows, K, rng, sf_lo=121, sf_hi=133):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    sf_log = rng.integers(sf_lo, sf_hi, size=(rows, K // 32), dtype=np.uint8)
    return codes, sf_log, oracle.sf_swizzle(sf_log, rows, K)


def _exact_value(codes, sf_log, r, k):
    byte = int(codes[r, k // 2])
    q = byte & 0xF if k % 2 == 0 else byte >> 4
    return E2M1[q] * Fraction(2) ** (int(sf_log[r, k // 32]) - 127)


@pytest.mark.parametrize("M,N,K", [(3, 2, 64), (5, 7, 160), (1, 1, 32)])
def test_gemm_exact_on_tiny_shapes(M, N, K):
    rng = np.random.default_rng(M * 100 + N * 10 + K)
    ac, asl, asf = _random_mx(M, K, rng)
    bc, bsl, bsf = _random_mx(N, K, rng)
    y = oracle.gemm(ac, asf, bc, bsf, M, N, K)
    for m in range(M):
        for n in range(N):
            want = sum(_exact_value(ac, asl, m, k) * _exact_value(bc, bsl, n, k) for k in range(K))
            assert Fraction(y[m, n]) == want, (m, n)


def test_gemm_alpha_bias_rows():
    rng = np.random.default_rng(1)
    M, N, K = 6, 5, 96
    ac, _, asf = _random_mx(M, K, rng)
    bc, _, bsf = _random_mx(N, K, rng)
    base = oracle.gemm(ac, asf, bc, bsf, M, N, K)
    bias = torch.tensor([0.5, -1.0, 3.0, 0.0, 1e3], dtype=torch.bfloat16)
    bias_bits = bias.view(torch.int16).numpy().view(np.uint16)
    y = oracle.gemm(ac, asf, bc, bsf, M, N, K, alpha=0.25, bias_bits=bias_bits, rows=np.array([4, 0, 5]))
    np.testing.assert_array_equal(y, 0.25 * base[[4, 0, 5]] + bias.double().numpy()[None, :])


def test_gemm_fp8_activation_exact():
    rng = np.random.default_rng(2)
    M, N, K = 3, 4, 64
    a8 = rng.integers(0, 256, size=(M, K), dtype=np.uint8)
    a8[(a8 & 0x7F) == 0x7F] = 0x38            # keep codes finite
    bc, bsl, bsf = _random_mx(N, K, rng)
    y = oracle.gemm(a8, None, bc, bsf, M, N, K, alpha=2.0, a_fp8=True)
    for m in range(M):
        for n in range(N):
            want = 2 * sum(Fraction(oracle.e4m3_decode(int(a8[m, k]))) * _exact_value(bc, bsl, n, k)
                           for k in range(K))
            assert Fraction(y[m, n]) == want


def test_gemm_identity_weights_reproduce_dequantised_rows():
    """B = identity (code 1.0 = 0x2 on the diagonal, scale byte 127) gives y = deq(A)."""
    rng = np.random.default_rng(4)
    M, K = 4, 64
    ac, _, asf = _random_mx(M, K, rng)
    N = K
    bc = np.zeros((N, K // 2), np.uint8)
    for n in range(N):
        bc[n, n // 2] = 0x2 << (4 * (n % 2))
    bsf = oracle.sf_swizzle(np.full((N, K // 32), 127, np.uint8), N, K)
    y = oracle.gemm(ac, asf, bc, bsf, M, N, K)
    np.testing.assert_array_equal(y, oracle.dequant_mxfp4(ac, asf, M, K))


def test_page_quadrature_table_is_quadrature():
    for name, w, a, both in golden("error_quadrature.txt"):
        w, a, both = float(w), float(a), float(both)
        assert abs(math.hypot(w, a) / both - 1) < 0.05, name
    row = golden("error_quadrature.txt")[0]
    # the page's 0.2074 comes from unrounded table entries: agree to 2e-4
    assert abs(math.hypot(float(row[1]), float(row[2])) - 0.2074) < 2e-4


def test_oracle_errors_add_in_quadrature():
    """Weight-only and activation-only MXFP4 errors combine in quadrature (+-10%)."""
    M, K, N = 128, 1024, 256
    x = inputs.normal_bf16(M, K, 1.0, seed=21)
    w = inputs.normal_bf16(N, K, 0.02, seed=22)
    ref = x.double().numpy() @ w.double().numpy().T
    ac, asl = oracle.quantize_mxfp4(x)
    bc, bsl = oracle.quantize_mxfp4(w)
    asf, bsf = oracle.sf_swizzle(asl, M, K), oracle.sf_swizzle(bsl, N, K)
    xq = oracle.dequant_mxfp4(ac, asf, M, K)
    wq = oracle.dequant_mxfp4(bc, bsf, N, K)

    def rel(y):
        return np.linalg.norm(y - ref) / np.linalg.norm(ref)

    e_w = rel(x.double().numpy() @ wq.T)
    e_a = rel(xq @ w.double().numpy().T)
    e_both = rel(oracle.gemm(ac, asf, bc, bsf, M, N, K))
    assert abs(math.hypot(e_w, e_a) / e_both - 1) < 0.10, (e_w, e_a, e_both)
    assert 0.05 < e_both < 0.3
