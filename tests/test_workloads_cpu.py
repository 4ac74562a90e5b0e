"""The benchmark's work counts and the seeded input generators (no GPU).

The roofline numbers divide by these counts, so each is checked against a
brute-force count: decode bytes (K and V of the live tokens, q, fp32 out) and
multi-token FLOPs (4 d per visible query-head/key pair, token j of sequence b
seeing L_b - n_b + j + 1 keys).
"""

import dataclasses

import numpy as np
import torch

from gqa_mqa_kv_b200 import workloads as W


def test_decode_bytes_count_live_rows_only():
    w = dataclasses.replace(W.WORKLOADS["llama2_70b_ragged"], B=5, seq_len=300)
    lens = W.seq_lens_for(w)
    brute = 0
    for b in range(w.B):
        for _t in range(int(lens[b])):
            brute += 2 * w.H_KV * w.D * 2  # one K row and one V row of every KV head, bf16
    brute += w.B * w.H_Q * w.D * 2 + w.B * w.H_Q * w.D * 4  # q (bf16) and out (fp32)
    assert W.algorithmic_bytes(w, lens) == brute
    w8 = dataclasses.replace(w, kv8=True)
    assert W.algorithmic_bytes(w8, lens) == brute - int(lens.sum()) * 2 * w.H_KV * w.D


def test_prefill_flops_count_visible_pairs():
    rng = np.random.default_rng(0)
    for _ in range(20):
        B = int(rng.integers(1, 5))
        n = rng.integers(0, 40, B)
        L = n + rng.integers(0, 60, B)
        w = W.PrefillWorkload("c", B, 8, 2, 128, 1, 0, seed=0)
        pairs = 0
        for b in range(B):
            for j in range(int(n[b])):
                pos = int(L[b]) - int(n[b]) + j
                pairs += sum(1 for t in range(int(L[b])) if t <= pos)
        assert W.prefill_flops(w, n, L) == 4 * w.D * w.H_Q * pairs


def test_prefill_workload_lengths():
    for w in W.PREFILL_WORKLOADS.values():
        n, L = W.prefill_lengths(w)
        assert n.shape == L.shape == (w.B,)
        assert (n >= 1).all() and (n <= w.q_len).all()
        assert ((L - n) >= 0).all() and ((L - n) <= w.prefix).all()
        if not w.ragged:
            assert (n == w.q_len).all() and (L == w.q_len + w.prefix).all()
        n2, L2 = W.prefill_lengths(w)
        assert (n == n2).all() and (L == L2).all()  # seeded


def test_prefill_inputs_layout():
    w = W.PrefillWorkload("c", 3, 8, 2, 16, 1, 0, seed=5, page_size=W.PAGE_SIZE)
    n, L = np.array([5, 0, 70]), np.array([9, 3, 130])
    inp = W.make_prefill_inputs(w, pad_value=float("nan"), lengths=(n, L))
    assert inp["q"].shape == (75, 8, 16) and inp["q"].dtype == torch.bfloat16
    assert inp["cu_q"].tolist() == [0, 5, 5, 75] and inp["max_q"] == 70
    assert inp["seq_lens"].tolist() == [9, 3, 130]
    k, v = inp["k"], inp["v"]
    assert k.shape[1] % W.PAGE_SIZE == 0 and k.shape[1] >= 130
    for b in range(3):
        assert torch.isfinite(k[b, : L[b]].float()).all() and torch.isnan(k[b, L[b]:].float()).all()
        assert torch.isnan(v[b, L[b]:].float()).all()
    # paged copy: token t of sequence b in page table[b, t // 64], slot t % 64
    table = inp["block_table"]
    for b in range(3):
        for t in (0, 63, 64, int(L[b]) - 1):
            if t < L[b]:
                assert torch.equal(inp["k_paged"][table[b, t // 64], t % 64], k[b, t])
                assert torch.equal(inp["v_paged"][table[b, t // 64], t % 64], v[b, t])
    # the same seed gives the same values
    again = W.make_prefill_inputs(w, pad_value=float("nan"), lengths=(n, L))
    assert torch.equal(again["q"], inp["q"]) and torch.equal(again["k"][0, :9], k[0, :9])
