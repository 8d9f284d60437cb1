"""Pins for the oracle's BF16 rounding and quantise-dequantise emulation."""

import struct

import numpy as np
import torch

import oracle
from mxfp4_block_scaled_mxq_b200 import inputs


def _bits(f):
    return struct.unpack("<I", struct.pack("<f", f))[0]


def test_bf16_rne_matches_torch_and_ties():
    rng = np.random.default_rng(0)
    vals = np.concatenate([rng.standard_normal(20000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 20000),
                           np.array([0.0, -0.0, 1e-45, -3e38, 3.3e38, 65504.0], np.float32)]).astype(np.float32)
    want = torch.from_numpy(vals).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_rne(float(v)) for v in vals], np.uint16)
    np.testing.assert_array_equal(got, want)
    # exact ties go to the even BF16 mantissa
    assert oracle.bf16_rne(struct.unpack("<f", struct.pack("<I", 0x3F808000))[0]) == 0x3F80
    assert oracle.bf16_rne(struct.unpack("<f", struct.pack("<I", 0x3F818000))[0]) == 0x3F82


def test_qdq_mxfp4_is_dequant_of_quant():
    x = inputs.heavy_tailed_bf16(40, 256, seed=12, token_fraction=0.1, token_factor=50.0)
    for rule in (oracle.RULE_OCP, oracle.RULE_UOS):
        for had in (False, True):
            out = oracle.qdq_mxfp4(x, rule=rule, hadamard=had)
            codes, sl = oracle.quantize_mxfp4(x, rule=rule, hadamard=had)
            deq = oracle.dequant_mxfp4(codes, oracle.sf_swizzle(sl, 40, 256), 40, 256)
            want = torch.from_numpy(deq).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
            np.testing.assert_array_equal(out, want)
            # every dequantised value is exactly a BF16 number (the E2M1 x 2^e product is exact)
            assert np.array_equal(torch.from_numpy(out.view(np.int16)).view(torch.bfloat16).double().numpy(), deq)


def test_qdq_fp8_recomposition():
    x, _, x_cal = inputs.flux_w4a8(M=16)
    s = inputs.static_fp8_scale(x_cal)
    out = oracle.qdq_fp8(x, s)
    q = oracle.quantize_fp8(x, s)
    dec = np.vectorize(oracle.e4m3_decode)(q).astype(np.float32) * np.float32(s)
    want = torch.from_numpy(dec.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(out, want)
