"""Pins for the oracle's 8-bit (E4M3) cache decoding and per-head scales (no GPU).

The E4M3 encoding follows the OCP 8-bit floating point definition (bias 7,
subnormals at exponent 0, S.1111.111 is NaN, no infinity, max 448).  The
scaled cache follows the bytes-per-element term of "Grouped-Query Attention
Shares Keys Without Sharing Every Query" (aitamer.news, the cache-estimate
paragraph): the same attention over keys and values stored in fewer bytes,
K = stored_k * k_scale[g], V = stored_v * v_scale[g].
"""

import math

import numpy as np
import pytest
import torch

import oracle

LANDMARKS = {
    0x00: 0.0, 0x80: -0.0, 0x38: 1.0, 0x40: 2.0, 0x30: 0.5, 0x3C: 1.5, 0xB8: -1.0,
    0x7E: 448.0, 0xFE: -448.0, 0x08: 2.0 ** -6, 0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9,
    0x77: 240.0, 0x78: 256.0,
}


def test_e4m3_landmark_values():
    t = oracle.e4m3_table()
    for byte, val in LANDMARKS.items():
        assert t[byte] == val, hex(byte)
        assert math.copysign(1.0, t[byte]) == math.copysign(1.0, val), hex(byte)
    assert math.isnan(t[0x7F]) and math.isnan(t[0xFF])
    assert np.sum(np.isnan(t)) == 2


def test_e4m3_table_matches_torch_float8():
    t = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(t))
    assert np.array_equal(t[~nan], ref[~nan])


def fp8_problem(B, H_Q, H_KV, D, S, lens, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H_Q, D, generator=g).to(torch.bfloat16)
    k = (torch.randn(B, S, H_KV, D, generator=g) * 40).to(torch.float8_e4m3fn)
    v = (torch.randn(B, S, H_KV, D, generator=g) * 40).to(torch.float8_e4m3fn)
    ks = torch.rand(H_KV, generator=g, dtype=torch.float64) / 40 + 0.01
    vs = torch.rand(H_KV, generator=g, dtype=torch.float64) / 40 + 0.01
    return q, k, v, ks, vs, torch.tensor(lens, dtype=torch.int32)


def test_scaled_decode_equals_plain_decode_on_dequantised_cache():
    q, k, v, ks, vs, L = fp8_problem(2, 8, 2, 16, 20, [20, 7], 1)
    got = oracle.gqa_decode_scaled(q, k, v, L, 0.25, ks, vs)
    kd = k.double() * ks[None, None, :, None]  # torch's own fp8 decoding and scaling
    vd = v.double() * vs[None, None, :, None]
    ref = oracle.gqa_decode(q, kd, vd, L, 0.25)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def test_unit_scales_equal_the_bf16_path_exactly():
    q, k, v, _, _, L = fp8_problem(2, 4, 1, 8, 9, [9, 3], 2)
    ones = np.ones(1)
    got = oracle.gqa_decode_scaled(q, k, v, L, 0.5, ones, ones)
    ref = oracle.gqa_decode(q, k.to(torch.bfloat16), v.to(torch.bfloat16), L, 0.5)  # E4M3 is exact in bf16
    assert np.array_equal(got, ref)


def test_scales_act_on_scores_and_values():
    q, k, v, ks, vs, L = fp8_problem(1, 4, 2, 8, 12, [12], 3)
    base = oracle.gqa_decode_scaled(q, k, v, L, 0.3, ks, vs)
    np.testing.assert_allclose(oracle.gqa_decode_scaled(q, k, v, L, 0.3, ks, vs * 2), 2 * base, rtol=1e-14)
    np.testing.assert_allclose(oracle.gqa_decode_scaled(q, k, v, L, 0.3, ks * 2, vs),
                               oracle.gqa_decode_scaled(q, k, v, L, 0.6, ks, vs), rtol=1e-12, atol=1e-14)
    # per-head: scaling only KV head 1 leaves the heads of group 0 unchanged
    vs2 = vs.clone()
    vs2[1] *= 3
    other = oracle.gqa_decode_scaled(q, k, v, L, 0.3, ks, vs2)
    assert np.array_equal(other[:, :2], base[:, :2])
    np.testing.assert_allclose(other[:, 2:], 3 * base[:, 2:], rtol=1e-14)
