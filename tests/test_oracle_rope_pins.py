"""Pins for the oracle's rotary position embedding (no GPU).

Source: "Grouped-Query Attention (GQA) and Multi-Query Attention (MQA):
Mathematical Foundations, Arithmetic Intensity, and KV-Cache Scaling
Mechanics" (llms.blog), section 4, "Rotary Position Embeddings (RoPE)
Interaction": R_{Theta,m} = diag(R_{theta_1,m}, ..., R_{theta_{d/2},m}), RoPE
applied to every query head and once to every key head, and the
relative-position identity <R_m q, R_n k> = q R_{m-n} k^T.

Each test ties the oracle to something other than its own formula: known
values of cos 1 and sin 1, a case whose only non-trivial rotation comes from
the second frequency (fixing the exponent of theta_i), torch complex128
multiplication, the page's relative-position identity, orthogonality,
composition of rotations, and the permutation between the two pairings.
"""

import math

import numpy as np
import pytest
import torch

import oracle

COS1, SIN1 = 0.5403023058681398, 0.8414709848078965  # cos(1 rad), sin(1 rad)


def rand(B, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(B, H, D, generator=g, dtype=torch.float64)


def test_position_zero_is_the_identity():
    x = rand(2, 3, 8, 1)
    out = oracle.rope(x, [0, 0])
    assert np.array_equal(out, x.numpy())


def test_single_pair_rotates_by_the_position():
    """d = 2: theta_1 = base^0 = 1, so position 1 rotates by exactly 1 rad."""
    out = oracle.rope(np.array([[[1.0, 0.0]]]), [1], base=12345.0)
    np.testing.assert_allclose(out[0, 0], [COS1, SIN1], rtol=0, atol=1e-15)
    out = oracle.rope(np.array([[[0.0, 1.0]]]), [1])
    np.testing.assert_allclose(out[0, 0], [-SIN1, COS1], rtol=0, atol=1e-15)


def test_second_frequency_is_base_to_the_minus_two_over_d():
    """d = 4, base 10^4: theta = (1, 10^-2).  At m = 100 the second pair turns
    by exactly 1 rad; a wrong exponent would turn it by something else."""
    out = oracle.rope(np.array([[[0.0, 0.0, 1.0, 0.0]]]), [100], base=10000.0)
    np.testing.assert_allclose(out[0, 0], [0.0, 0.0, COS1, SIN1], rtol=0, atol=1e-13)
    out = oracle.rope(np.array([[[1.0, 0.0, 0.0, 0.0]]]), [100], base=10000.0)
    np.testing.assert_allclose(out[0, 0, :2], [math.cos(100.0), math.sin(100.0)], rtol=0, atol=1e-13)


def test_matches_complex_multiplication():
    D, base = 16, 10000.0
    x = rand(2, 4, D, 2)
    pos = [7, 1234]
    out = oracle.rope(x, pos, base=base)
    z = torch.complex(x[..., 0::2], x[..., 1::2])  # adjacent pairs as complex numbers
    inv = torch.tensor([base ** (-2.0 * i / D) for i in range(D // 2)], dtype=torch.float64)
    ang = torch.tensor(pos, dtype=torch.float64)[:, None, None] * inv
    zr = z * torch.polar(torch.ones_like(ang), ang)
    ref = torch.stack([zr.real, zr.imag], dim=-1).reshape(x.shape)
    np.testing.assert_allclose(out, ref.numpy(), rtol=0, atol=1e-12)


@pytest.mark.parametrize("m,n", [(5, 3), (3, 5), (1000, 0), (77, 77), (131071, 12)])
def test_relative_position_identity(m, n):
    """<R_m q, R_n k> = <R_{m-n} q, k>  ([LLMS] section 4)."""
    q = rand(1, 1, 64, 3)
    k = rand(1, 1, 64, 4)
    lhs = float(np.dot(oracle.rope(q, [m])[0, 0], oracle.rope(k, [n])[0, 0]))
    d = m - n
    if d >= 0:
        rhs = float(np.dot(oracle.rope(q, [d])[0, 0], k[0, 0].numpy()))
    else:
        rhs = float(np.dot(q[0, 0].numpy(), oracle.rope(k, [-d])[0, 0]))
    assert lhs == pytest.approx(rhs, rel=1e-9, abs=1e-9)


def test_rotation_preserves_every_pair_norm():
    x = rand(3, 2, 32, 5)
    out = oracle.rope(x, [9, 4000, 65535])
    pn_in = x.numpy().reshape(3, 2, 16, 2)
    pn_out = out.reshape(3, 2, 16, 2)
    np.testing.assert_allclose(np.hypot(pn_out[..., 0], pn_out[..., 1]),
                               np.hypot(pn_in[..., 0], pn_in[..., 1]), rtol=1e-13, atol=0)


def test_rotations_compose():
    x = rand(1, 2, 16, 6)
    once = oracle.rope(x, [300])
    twice = oracle.rope(oracle.rope(x, [100]), [200])
    np.testing.assert_allclose(twice, once, rtol=0, atol=1e-12)


def test_halves_pairing_is_adjacent_pairing_up_to_a_permutation():
    D = 16
    x = rand(2, 3, D, 7)
    perm = np.stack([np.arange(D // 2), np.arange(D // 2) + D // 2], axis=1).reshape(-1)  # i, i+D/2 adjacent
    adj = oracle.rope(x.numpy()[..., perm], [11, 5000], pairing="adjacent")
    half = oracle.rope(x, [11, 5000], pairing="halves")
    np.testing.assert_allclose(half[..., perm], adj, rtol=0, atol=1e-14)


def test_rows_rotate_by_their_own_position():
    x = rand(2, 1, 8, 8)
    both = oracle.rope(x, [3, 40])
    assert np.array_equal(both[0], oracle.rope(x[:1], [3])[0])
    assert np.array_equal(both[1], oracle.rope(x[1:], [40])[0])


def test_bf16_input_widens_exactly():
    x = rand(1, 2, 8, 9).to(torch.bfloat16)
    assert np.array_equal(oracle.rope(x, [17]), oracle.rope(x.double(), [17]))


def test_rejects_odd_head_dim():
    with pytest.raises(ValueError):
        oracle.rope(np.zeros((1, 1, 3)), [1])
