"""Pins for the fp64 CPU oracle (no GPU).

Each test ties the oracle to something other than itself: values the pages
print, closed forms, special cases that reduce to a library routine
(torch's scaled_dot_product_attention in float64, torch.repeat_interleave,
torch.logsumexp), and brute force on tiny inputs.  Together they are chosen so
that a plausible slip in the oracle -- a dropped scale, a wrong sign in the
exponent, a strided instead of contiguous group map, an off-by-one token
bound, swapped K/V operands, a wrong batch stride, a lossy bf16 widening, a
wrong LSE merge -- fails at least one of them.

Sources:
  [LLMS] "Grouped-Query Attention (GQA) and Multi-Query Attention (MQA):
         Mathematical Foundations, Arithmetic Intensity, and KV-Cache Scaling
         Mechanics" (llms.blog)
  [AIT]  "Grouped-Query Attention Shares Keys Without Sharing Every Query"
         (aitamer.news)
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rand_problem(B, H_Q, H_KV, D, S_max, lens, seed, dtype=torch.float64, pad=0.0):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H_Q, D, generator=g, dtype=torch.float64).to(dtype)
    k = torch.randn(B, S_max, H_KV, D, generator=g, dtype=torch.float64).to(dtype)
    v = torch.randn(B, S_max, H_KV, D, generator=g, dtype=torch.float64).to(dtype)
    for b, L in enumerate(lens):
        k[b, L:] = pad
        v[b, L:] = pad
    return q, k, v, torch.tensor(lens, dtype=torch.int32)


def sdpa_reference(q, k, v, lens, scale, gqa=True):
    """torch SDPA in float64, one batch row at a time (library routine)."""
    B, H_Q, D = q.shape
    out = torch.zeros(B, H_Q, D, dtype=torch.float64)
    for b in range(B):
        L = int(lens[b])
        if L == 0:
            continue
        qb = q[b].double().unsqueeze(0).unsqueeze(2)  # [1, H_Q, 1, D]
        kb = k[b, :L].double().permute(1, 0, 2).unsqueeze(0)  # [1, H_KV, L, D]
        vb = v[b, :L].double().permute(1, 0, 2).unsqueeze(0)
        o = F.scaled_dot_product_attention(qb, kb, vb, scale=scale, enable_gqa=gqa)
        out[b] = o[0, :, 0, :]
    return out


# ----------------------------------------------------------------------------
# KV-cache size formula: [LLMS] section 1 table, [AIT] cache-estimate paragraph
# ----------------------------------------------------------------------------

def test_kv_cache_bytes_matches_printed_table():
    with open(os.path.join(GOLDEN, "kv_cache_table_70b.json")) as f:
        gold = json.load(f)
    m = gold["model"]
    cols = {"MHA_H_KV_64": 64, "GQA8_H_KV_8": 8, "MQA_H_KV_1": 1}
    for row in gold["rows"]:
        for col, h_kv in cols.items():
            gb = oracle.kv_cache_bytes(m["layers"], row["tokens"], h_kv, m["d_k"], m["elem_bytes"]) / 1e9
            assert round(gb, 2) == pytest.approx(row[col], abs=1e-9), (row, col, gb)
    pc = gold["prose_checks"]
    mha = oracle.kv_cache_bytes(80, 131072, 64, 128, 2)
    gqa = oracle.kv_cache_bytes(80, 131072, 8, 128, 2)
    assert round(mha / 1e9, 1) == pc["mha_131072_GB"]
    assert mha / gqa == pc["gqa8_reduction_factor"]


def test_cache_element_ratios():
    with open(os.path.join(GOLDEN, "cache_element_ratios.json")) as f:
        gold = json.load(f)
    mha = oracle.kv_cache_bytes(1, 1, gold["H_Q"], 128, 2)
    for case in gold["cases"]:
        num, den = case["ratio_to_mha"]
        assert oracle.kv_cache_bytes(1, 1, case["H_KV"], 128, 2) * den == mha * num


def test_kv_cache_bytes_scales_with_every_factor():
    base = oracle.kv_cache_bytes(2, 3, 5, 7, 2)
    assert base == 2 * 2 * 3 * 5 * 7 * 2
    assert oracle.kv_cache_bytes(2, 3, 5, 7, 1) * 2 == base  # bytes per element ([AIT])


# ----------------------------------------------------------------------------
# Attention: library special cases ([LLMS] section 2)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize(
    "B,H_Q,H_KV,D,lens",
    [
        (3, 8, 2, 16, [5, 17, 1]),     # GQA, R=4, ragged
        (2, 8, 8, 8, [9, 3]),          # MHA (G = H_Q)
        (2, 8, 1, 8, [7, 12]),         # MQA (G = 1)
        (1, 6, 3, 4, [11]),            # R=2, odd head count
        (2, 32, 1, 16, [33, 2]),       # MQA with R = 32
        (2, 12, 4, 8, [0, 6]),         # an empty sequence
    ],
)
def test_matches_torch_sdpa(B, H_Q, H_KV, D, lens):
    S_max = max(max(lens), 1) + 3
    scale = 0.37
    q, k, v, L = rand_problem(B, H_Q, H_KV, D, S_max, lens, seed=B * 100 + H_Q + H_KV)
    got = oracle.gqa_decode(q, k, v, L, scale)
    ref = sdpa_reference(q, k, v, L, scale)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_mha_case_is_plain_per_head_attention():
    """G = H_Q reduces to MHA ([LLMS] section 2): SDPA without any grouping."""
    q, k, v, L = rand_problem(2, 4, 4, 8, 10, [10, 6], seed=7)
    got = oracle.gqa_decode(q, k, v, L, 0.5)
    ref = sdpa_reference(q, k, v, L, 0.5, gqa=False)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_mqa_case_broadcasts_single_kv_head():
    """G = 1 reduces to MQA: K and V broadcast to every query head ([LLMS] section 2, MQA)."""
    q, k, v, L = rand_problem(2, 6, 1, 8, 9, [9, 4], seed=8)
    got = oracle.gqa_decode(q, k, v, L, 0.3)
    kx = k.expand(-1, -1, 6, -1).contiguous()  # broadcast, not a copy of the oracle's map
    vx = v.expand(-1, -1, 6, -1).contiguous()
    ref = sdpa_reference(q, kx, vx, L, 0.3, gqa=False)
    np.testing.assert_allclose(got, ref.numpy(), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("H_Q,H_KV", [(8, 2), (8, 4), (12, 3), (32, 1), (8, 8)])
def test_gqa_equals_mha_on_repeat_interleaved_kv(H_Q, H_KV):
    """[LLMS] section 2: K~ = repeat_interleave(K, R, dim=2), same for V.

    Same summation order on both sides, so the fp64 results agree exactly.
    """
    R = H_Q // H_KV
    q, k, v, L = rand_problem(2, H_Q, H_KV, 8, 13, [13, 5], seed=H_Q * 10 + H_KV)
    got = oracle.gqa_decode(q, k, v, L, 0.25)
    kr = torch.repeat_interleave(k, R, dim=2)
    vr = torch.repeat_interleave(v, R, dim=2)
    ref = oracle.gqa_decode(q, kr, vr, L, 0.25)
    assert np.array_equal(got, ref)


def test_group_map_is_contiguous():
    """Query head h reads KV head h // R, not h % H_KV ([LLMS] section 2, g(i))."""
    B, H_Q, H_KV, D, S = 2, 12, 3, 4, 5
    R = H_Q // H_KV
    q, k, _, L = rand_problem(B, H_Q, H_KV, D, S, [5, 3], seed=3)
    v = torch.zeros(B, S, H_KV, D, dtype=torch.float64)
    for g in range(H_KV):
        v[:, :, g, :] = g
    out = oracle.gqa_decode(q, k, v, L, 1.0)
    for h in range(H_Q):
        np.testing.assert_allclose(out[:, h, :], h // R, rtol=0, atol=1e-14)
    assert any((h // R) != (h % H_KV) for h in range(H_Q))


# ----------------------------------------------------------------------------
# Closed forms and hand-worked cases (softmax definition, [LLMS] section 2)
# ----------------------------------------------------------------------------

def test_length_one_returns_v_exactly():
    q, k, v, L = rand_problem(3, 8, 2, 8, 4, [1, 1, 1], seed=11, pad=5.0)
    out = oracle.gqa_decode(q, k, v, L, 0.7)
    for b in range(3):
        for h in range(8):
            assert np.array_equal(out[b, h], v[b, 0, h // 4].numpy())


def test_weights_sum_to_one_and_are_positive():
    q, k, _, L = rand_problem(2, 8, 2, 16, 40, [40, 23], seed=12)
    for b in range(2):
        for h in range(8):
            w = oracle.attention_weights(q, k, L, 0.25, b, h)
            assert w.shape == (int(L[b]),)
            assert np.all(w > 0)
            assert abs(w.sum() - 1.0) <= 1e-12


def test_weights_match_library_softmax():
    q, k, _, L = rand_problem(1, 4, 2, 8, 9, [9], seed=13)
    w = oracle.attention_weights(q, k, L, 0.5, 0, 3)
    s = (k[0, :, 1, :] @ q[0, 3]) * 0.5
    np.testing.assert_allclose(w, torch.softmax(s, dim=0).numpy(), rtol=1e-13, atol=0)


def test_identical_keys_give_mean_of_v():
    B, H_Q, H_KV, D, S = 2, 4, 2, 8, 17
    q, _, v, L = rand_problem(B, H_Q, H_KV, D, S, [17, 6], seed=14)
    g = torch.Generator().manual_seed(99)
    k = torch.randn(B, 1, H_KV, D, generator=g, dtype=torch.float64).expand(B, S, H_KV, D).contiguous()
    out = oracle.gqa_decode(q, k, v, L, 0.9)
    for b in range(B):
        for h in range(H_Q):
            mean = v[b, : int(L[b]), h // 2, :].mean(dim=0).numpy()
            np.testing.assert_allclose(out[b, h], mean, rtol=0, atol=1e-14)


def test_hand_computed_two_token_case():
    """Scores {0, ln 3} give weights {1/4, 3/4}."""
    q = torch.tensor([[[1.0, 0.0]]], dtype=torch.float64)            # [1,1,2]
    k = torch.tensor([[[[0.0, 5.0]], [[1.0, 7.0]]]], dtype=torch.float64)  # [1,2,1,2]
    v = torch.tensor([[[[4.0, 0.0]], [[0.0, 8.0]]]], dtype=torch.float64)
    L = torch.tensor([2], dtype=torch.int32)
    out = oracle.gqa_decode(q, k, v, L, math.log(3.0))
    np.testing.assert_allclose(out[0, 0], [1.0, 6.0], rtol=0, atol=1e-14)
    w = oracle.attention_weights(q, k, L, math.log(3.0), 0, 0)
    np.testing.assert_allclose(w, [0.25, 0.75], rtol=0, atol=1e-15)


def test_hand_computed_three_token_case_with_grouping():
    """Two query heads share one KV head; scores {0, ln 2, ln 5} -> {1/8, 2/8, 5/8}
    for head 0, and the sign-flipped query gives {1/(1+1/2+1/5)...} for head 1."""
    q = torch.tensor([[[1.0], [-1.0]]], dtype=torch.float64)  # [1, H_Q=2, D=1]
    k = torch.tensor([[[[0.0]], [[math.log(2.0)]], [[math.log(5.0)]]]], dtype=torch.float64)
    v = torch.tensor([[[[8.0]], [[16.0]], [[-8.0]]]], dtype=torch.float64)
    L = torch.tensor([3], dtype=torch.int32)
    out = oracle.gqa_decode(q, k, v, L, 1.0)
    assert out[0, 0, 0] == pytest.approx((8 * 1 + 16 * 2 - 8 * 5) / 8.0, abs=1e-14)
    z = 1 + 0.5 + 0.2
    assert out[0, 1, 0] == pytest.approx((8 * 1 + 16 * 0.5 - 8 * 0.2) / z, abs=1e-14)


def test_scale_enters_the_exponent():
    """Doubling scale equals doubling the query."""
    q, k, v, L = rand_problem(1, 4, 2, 8, 10, [10], seed=15)
    a = oracle.gqa_decode(q, k, v, L, 0.6)
    b = oracle.gqa_decode(q * 2, k, v, L, 0.3)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)
    c = oracle.gqa_decode(q, k, v, L, 0.3)
    assert np.max(np.abs(a - c)) > 1e-3


def test_one_hot_spike_selects_that_token():
    B, H_Q, H_KV, D, S = 2, 8, 2, 8, 70
    q = torch.ones(B, H_Q, D, dtype=torch.float64)
    k = torch.zeros(B, S, H_KV, D, dtype=torch.float64)
    g = torch.Generator().manual_seed(16)
    v = torch.randn(B, S, H_KV, D, generator=g, dtype=torch.float64)
    spikes = {(0, 0): 63, (0, 1): 0, (1, 0): 64, (1, 1): 69}
    for (b, g_), t in spikes.items():
        k[b, t, g_, :] = 100.0 / D
    L = torch.tensor([70, 70], dtype=torch.int32)
    out = oracle.gqa_decode(q, k, v, L, 1.0)
    for h in range(H_Q):
        for b in range(B):
            t = spikes[(b, h // 4)]
            np.testing.assert_allclose(out[b, h], v[b, t, h // 4].numpy(), rtol=0, atol=1e-30 + 1e-40)


def test_tokens_past_seq_len_are_never_read():
    lens = [5, 1, 9]
    qn, kn, vn, L = rand_problem(3, 4, 2, 8, 12, lens, seed=17, pad=float("nan"))
    q0, k0, v0, _ = rand_problem(3, 4, 2, 8, 12, lens, seed=17, pad=0.0)
    a = oracle.gqa_decode(qn, kn, vn, L, 0.4)
    b = oracle.gqa_decode(q0, k0, v0, L, 0.4)
    assert np.all(np.isfinite(a))
    assert np.array_equal(a, b)


def test_zero_length_sequence_gives_zero():
    q, k, v, L = rand_problem(2, 4, 2, 8, 6, [0, 6], seed=18)
    out = oracle.gqa_decode(q, k, v, L, 0.4)
    assert np.all(out[0] == 0.0)
    assert np.any(out[1] != 0.0)


def test_batch_rows_are_independent():
    q, k, v, L = rand_problem(3, 4, 2, 8, 7, [7, 4, 6], seed=19)
    full = oracle.gqa_decode(q, k, v, L, 0.5)
    for b in range(3):
        one = oracle.gqa_decode(q[b:b + 1], k[b:b + 1], v[b:b + 1], L[b:b + 1], 0.5)
        assert np.array_equal(one[0], full[b])


def test_brute_force_small_integers():
    """Enumerate small integer inputs; compare with the un-shifted softmax
    computed from math.exp in exact-order Python (tiny sizes only)."""
    rng = np.random.default_rng(20)
    for trial in range(200):
        L = int(rng.integers(1, 5))
        qv = rng.integers(-2, 3, size=(1, 2, 2)).astype(np.float64)
        kv = rng.integers(-2, 3, size=(1, L, 1, 2)).astype(np.float64)
        vv = rng.integers(-3, 4, size=(1, L, 1, 2)).astype(np.float64)
        out = oracle.gqa_decode(qv, kv, vv, [L], 0.5)
        for h in range(2):
            e = [math.exp(0.5 * (qv[0, h, 0] * kv[0, t, 0, 0] + qv[0, h, 1] * kv[0, t, 0, 1])) for t in range(L)]
            z = sum(e)
            for i in range(2):
                ref = sum(e[t] * vv[0, t, 0, i] for t in range(L)) / z
                assert out[0, h, i] == pytest.approx(ref, rel=1e-13, abs=1e-13)


def test_explicit_pairs_match_full_output():
    q, k, v, L = rand_problem(3, 8, 2, 8, 9, [9, 2, 5], seed=21)
    full = oracle.gqa_decode(q, k, v, L, 0.5)
    pairs = [(2, 7), (0, 0), (1, 3), (2, 4)]
    part = oracle.gqa_decode(q, k, v, L, 0.5, pairs=pairs)
    for j, (b, h) in enumerate(pairs):
        assert np.array_equal(part[j], full[b, h])


# ----------------------------------------------------------------------------
# Input widening
# ----------------------------------------------------------------------------

def test_bf16_and_f32_widen_exactly():
    q, k, v, L = rand_problem(2, 8, 2, 16, 11, [11, 7], seed=22, dtype=torch.bfloat16)
    a = oracle.gqa_decode(q, k, v, L, 0.25)
    b = oracle.gqa_decode(q.double(), k.double(), v.double(), L, 0.25)
    assert np.array_equal(a, b)
    c = oracle.gqa_decode(q.float(), k.float(), v.float(), L, 0.25)
    assert np.array_equal(a, c)


# ----------------------------------------------------------------------------
# Split-KV partials and the log-sum-exp merge
# ----------------------------------------------------------------------------

def test_partial_lse_matches_library_logsumexp():
    q, k, v, L = rand_problem(1, 4, 2, 8, 30, [30], seed=23)
    s = (k[0, 5:19, 1, :] @ q[0, 2]) * 0.5
    lse, o = oracle.partial(q, k, v, L, 0.5, 0, 2, 5, 19)
    assert lse == pytest.approx(float(torch.logsumexp(s, 0)), rel=1e-14)
    w = torch.softmax(s, 0)
    np.testing.assert_allclose(o, (w @ v[0, 5:19, 1, :]).numpy(), rtol=1e-13, atol=1e-14)


def test_split_then_combine_equals_unsplit():
    q, k, v, L = rand_problem(2, 8, 2, 16, 200, [200, 77], seed=24)
    full = oracle.gqa_decode(q, k, v, L, 0.3)
    rng = np.random.default_rng(25)
    for b in range(2):
        for h in range(8):
            Lb = int(L[b])
            cuts = sorted(set(rng.integers(0, Lb + 40, size=int(rng.integers(1, 7))).tolist()))
            bounds = [0] + cuts + [Lb + 64]
            parts = [oracle.partial(q, k, v, L, 0.3, b, h, bounds[i], bounds[i + 1])
                     for i in range(len(bounds) - 1)]
            lse = [p[0] for p in parts]
            o = np.stack([p[1] for p in parts])
            merged = oracle.lse_combine(lse, o)
            np.testing.assert_allclose(merged, full[b, h], rtol=0, atol=1e-12)


def test_combine_of_all_empty_partials_is_zero():
    out = oracle.lse_combine([-math.inf, -math.inf], np.zeros((2, 4)))
    assert np.all(out == 0.0)


def test_combine_weights_by_exp_lse():
    """Two partials with lse {0, ln 3} weigh {1/4, 3/4}."""
    out = oracle.lse_combine([0.0, math.log(3.0)], np.array([[4.0, 0.0], [0.0, 8.0]]))
    np.testing.assert_allclose(out, [1.0, 6.0], rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------
# Argument checks
# ----------------------------------------------------------------------------

def test_rejects_non_divisible_heads():
    q, k, v, L = rand_problem(1, 6, 4, 4, 3, [3], seed=26)
    with pytest.raises(ValueError):
        oracle.gqa_decode(q, k, v, L, 1.0)


def test_rejects_length_beyond_capacity():
    q, k, v, _ = rand_problem(1, 4, 2, 4, 3, [3], seed=27)
    with pytest.raises(ValueError):
        oracle.gqa_decode(q, k, v, torch.tensor([4], dtype=torch.int32), 1.0)
