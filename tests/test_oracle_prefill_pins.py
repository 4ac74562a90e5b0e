"""Pins of the oracle's multi-token (prefill) attention against facts outside it (no GPU).

The definition pinned here: query token j of sequence b sits at position
p = L_b - n_b + j and sees cache positions t <= p -- the causal mask M of
"Grouped-Query Attention (GQA) and Multi-Query Attention (MQA): Mathematical
Foundations, ..." section 2 (M[j][t] = 0 for t <= j, -inf after), shifted by
the cached prefix.  Each pin ties one part of that to a closed form, a
library routine or an invariant, so that a wrong position, an off-by-one in
the mask, a wrong sequence lookup or a transposed group map fails one of
them.
"""

import math

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def _case(B, H_Q, H_KV, D, n, prefix, seed, dtype=torch.float64, S_extra=3):
    """q packed [total_q, H_Q, D]; caches [B, S_max, H_KV, D]; L_b = prefix_b + n_b."""
    g = torch.Generator().manual_seed(seed)
    n = list(n)
    lens = [p + m for p, m in zip(prefix, n)]
    cu = np.concatenate([[0], np.cumsum(n)]).astype(np.int32)
    S_max = max(lens) + S_extra
    q = torch.randn(int(cu[-1]), H_Q, D, generator=g, dtype=torch.float64).to(dtype)
    k = torch.randn(B, S_max, H_KV, D, generator=g, dtype=torch.float64).to(dtype)
    v = torch.randn(B, S_max, H_KV, D, generator=g, dtype=torch.float64).to(dtype)
    return q, k, v, np.array(lens, dtype=np.int32), cu


def test_first_token_of_a_fresh_prompt_returns_its_own_value():
    # Position 0 sees only key 0: the weight is exactly 1.
    q, k, v, lens, cu = _case(3, 6, 2, 16, n=[5, 1, 7], prefix=[0, 0, 0], seed=1)
    out = oracle.gqa_prefill(q, k, v, lens, cu, 0.37)
    R = 3
    for b in range(3):
        for h in range(6):
            np.testing.assert_array_equal(out[cu[b], h], v[b, 0, h // R].numpy())


def test_equal_keys_give_the_mean_of_the_visible_values():
    # All keys of a (b, g) equal -> every visible score equal -> weights 1/(p+1):
    # out = mean of V over positions 0..p.  Pins the position p = L_b - n_b + j.
    B, H_Q, H_KV, D = 3, 8, 2, 8
    q, k, v, lens, cu = _case(B, H_Q, H_KV, D, n=[4, 6, 3], prefix=[5, 0, 9], seed=2)
    k[:] = k[:, :1].clone()  # broadcast position 0's key to every position
    out = oracle.gqa_prefill(q, k, v, lens, cu, 0.5)
    vn = v.numpy()
    R = H_Q // H_KV
    for b in range(B):
        n_b = cu[b + 1] - cu[b]
        for j in range(n_b):
            p = lens[b] - n_b + j
            for h in range(H_Q):
                want = vn[b, : p + 1, h // R].mean(axis=0)
                np.testing.assert_allclose(out[cu[b] + j, h], want, rtol=0, atol=1e-13)


def _sdpa_reference(q, k, v, lens, cu, scale, R, is_causal=False):
    """torch's scaled_dot_product_attention in float64, one sequence at a time."""
    outs = []
    for b in range(len(lens)):
        n_b, L = int(cu[b + 1] - cu[b]), int(lens[b])
        qb = q[cu[b]: cu[b + 1]].permute(1, 0, 2)                       # [H_Q, n_b, D]
        kb = k[b, :L].permute(1, 0, 2).repeat_interleave(R, dim=0)      # [H_Q, L, D]
        vb = v[b, :L].permute(1, 0, 2).repeat_interleave(R, dim=0)
        if is_causal:
            assert n_b == L
            ob = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, is_causal=True, scale=scale)
        else:
            pos = torch.arange(n_b)[:, None] + (L - n_b)
            mask = torch.arange(L)[None, :] <= pos                     # True = attend
            ob = torch.nn.functional.scaled_dot_product_attention(qb, kb, vb, attn_mask=mask, scale=scale)
        outs.append(ob.permute(1, 0, 2))
    return torch.cat(outs).numpy()


@pytest.mark.parametrize("H_Q,H_KV", [(8, 2), (6, 6), (4, 1), (12, 4)])
def test_matches_library_attention_with_an_explicit_prefix_mask(H_Q, H_KV):
    q, k, v, lens, cu = _case(3, H_Q, H_KV, 16, n=[5, 2, 9], prefix=[3, 11, 0], seed=3)
    out = oracle.gqa_prefill(q, k, v, lens, cu, 0.25)
    ref = _sdpa_reference(q, k, v, lens, cu, 0.25, H_Q // H_KV)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_fresh_prompts_match_library_causal_attention():
    # No prefix: the library builds the s x s causal mask itself.
    q, k, v, lens, cu = _case(2, 8, 4, 32, n=[13, 7], prefix=[0, 0], seed=4, S_extra=0)
    out = oracle.gqa_prefill(q, k, v, lens, cu, 1 / math.sqrt(32))
    ref = _sdpa_reference(q, k, v, lens, cu, 1 / math.sqrt(32), 2, is_causal=True)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_no_token_reads_a_later_position():
    # NaN planted at every position after p0 leaves tokens up to p0 untouched and
    # finite; the token just after sees it.
    q, k, v, lens, cu = _case(1, 4, 2, 8, n=[10], prefix=[4], seed=5)
    base = oracle.gqa_prefill(q, k, v, lens, cu, 0.3)
    j0 = 5
    p0 = int(lens[0]) - 10 + j0
    k2, v2 = k.clone(), v.clone()
    k2[0, p0 + 1:] = float("nan")
    v2[0, p0 + 1:] = float("nan")
    out = oracle.gqa_prefill(q, k2, v2, lens, cu, 0.3)
    np.testing.assert_array_equal(out[: j0 + 1], base[: j0 + 1])
    assert np.isnan(out[j0 + 1:]).all()


def test_rows_map_to_their_sequence_and_heads_to_their_group():
    # V constant per (b, g): every output row equals 10 b + g + 1 whatever the
    # weights, so a wrong span lookup or a strided group map shows.  One
    # sequence brings no tokens.
    B, H_Q, H_KV, D = 4, 8, 4, 8
    q, k, v, lens, cu = _case(B, H_Q, H_KV, D, n=[3, 0, 5, 2], prefix=[2, 4, 0, 7], seed=6)
    for b in range(B):
        for g_ in range(H_KV):
            v[b, :, g_] = 10 * b + g_ + 1
    out = oracle.gqa_prefill(q, k, v, lens, cu, 0.4)
    R = H_Q // H_KV
    for b in range(B):
        for i in range(cu[b], cu[b + 1]):
            for h in range(H_Q):
                np.testing.assert_allclose(out[i, h], 10 * b + h // R + 1, rtol=1e-14)


def test_one_token_per_sequence_is_the_decode_step():
    # n_b = 1: the token sits at L_b - 1 and sees the whole cache (the decode
    # oracle, pinned by its own suite).
    B, H_Q, H_KV, D = 3, 8, 2, 16
    q, k, v, lens, cu = _case(B, H_Q, H_KV, D, n=[1, 1, 1], prefix=[6, 0, 12], seed=7)
    out = oracle.gqa_prefill(q, k, v, lens, cu, 0.2)
    dec = oracle.gqa_decode(q, k, v, lens, 0.2)
    np.testing.assert_allclose(out, dec, rtol=1e-13, atol=1e-14)


def test_bf16_inputs_widen_exactly():
    q, k, v, lens, cu = _case(2, 4, 2, 16, n=[3, 4], prefix=[1, 2], seed=8, dtype=torch.bfloat16)
    out = oracle.gqa_prefill(q, k, v, lens, cu, 0.25)
    ref = _sdpa_reference(q.double(), k.double(), v.double(), lens, cu, 0.25, 2)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_listed_rows_equal_the_full_result():
    q, k, v, lens, cu = _case(2, 8, 2, 16, n=[6, 3], prefix=[2, 5], seed=9)
    full = oracle.gqa_prefill(q, k, v, lens, cu, 0.3)
    rows = [(0, 0), (5, 7), (6, 3), (8, 1)]
    part = oracle.gqa_prefill(q, k, v, lens, cu, 0.3, rows=rows)
    for r, (i, h) in enumerate(rows):
        np.testing.assert_array_equal(part[r], full[i, h])


@pytest.mark.parametrize("cu,lens", [([1, 3, 5], [4, 4]),      # cu_q[0] != 0
                                     ([0, 3, 2], [4, 4]),      # decreasing
                                     ([0, 5, 7], [4, 4])])     # n_b > L_b
def test_rejects_inconsistent_spans(cu, lens):
    q = torch.zeros(cu[-1] if cu[-1] > 0 else 1, 2, 8, dtype=torch.float64)
    k = torch.zeros(2, 6, 1, 8, dtype=torch.float64)
    with pytest.raises(ValueError):
        oracle.gqa_prefill(q[: max(cu[-1], 0)], k, k, lens, cu, 0.5)
