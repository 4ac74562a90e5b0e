"""Parity of the multi-token (prefill) kernel with the fp64 oracle (GPU).

Query token j of sequence b sits at position L_b - n_b + j and attends to
cache positions t <= it ("Grouped-Query Attention (GQA) and Multi-Query
Attention (MQA): Mathematical Foundations, ...", section 2, Head_i with the
causal mask M).  Small cases are compared element by element; the benchmark
workloads at full size on sampled (row, head) outputs.  Tolerance as for
decode (tests/helpers.py).  Cache rows at or past L_b hold NaN in every case
to prove they never reach an output.
"""

import numpy as np
import pytest
import torch

import oracle
from gqa_mqa_kv_b200 import FLAG_BAD_QUERY_SPAN, gqa_prefill, make_params, make_workspace, read_status
from gqa_mqa_kv_b200 import workloads as W
from helpers import assert_parity

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _workload(B, H_Q, H_KV, page=0, seed=21):
    return W.PrefillWorkload("case", B, H_Q, H_KV, 128, 1, 0, seed=seed, page_size=page)


def _run(inp, w, out_dtype=torch.float32, max_q=None, cu=None):
    paged = w.page_size > 0
    k = (inp["k_paged"] if paged else inp["k"]).to(DEV)
    v = (inp["v_paged"] if paged else inp["v"]).to(DEV)
    bt = inp["block_table"].to(DEV) if paged else None
    lens = inp["seq_lens"].to(DEV)
    cu_q = (inp["cu_q"] if cu is None else cu).to(DEV)
    q = inp["q"].to(DEV)
    proxy = torch.empty((w.B, w.H_Q, w.D), dtype=torch.bfloat16, device="meta")
    ws = torch.zeros_like(make_workspace(make_params(proxy, k, lens, bt), DEV))
    out = gqa_prefill(q, k, v, lens, cu_q, max_q_len=inp["max_q"] if max_q is None else max_q,
                      block_table=bt, out_dtype=out_dtype, workspace=ws,
                      )
    torch.cuda.synchronize()
    return out, read_status(ws)


def _case(B, H_Q, H_KV, n, prefix, page=0, seed=21):
    w = _workload(B, H_Q, H_KV, page, seed)
    n = np.asarray(n, dtype=np.int32)
    lens = n + np.asarray(prefix, dtype=np.int32)
    return w, W.make_prefill_inputs(w, pad_value=float("nan"), lengths=(n, lens))


def _oracle(inp, w, rows=None):
    return oracle.gqa_prefill(inp["q"], inp["k"], inp["v"], inp["seq_lens"], inp["cu_q"], w.softmax_scale,
                              rows=rows)


# n: a fresh prompt over two key steps, one decode-like token after a prefix, a
# ragged middle, and a sequence with no new tokens.
N_MIX, PREFIX_MIX = [200, 1, 77, 0], [0, 300, 50, 9]


@pytest.mark.parametrize("R", [1, 3, 4, 8, 16, 32, 64])
def test_parity_contiguous(R):
    w, inp = _case(4, 2 * R, 2, N_MIX, PREFIX_MIX, seed=30 + R)
    out, flags = _run(inp, w)
    assert flags == 0
    assert_parity(out.cpu(), _oracle(inp, w), f"prefill R={R}")


def test_parity_one_token_per_row_group_of_128_heads():
    # R = 128: a tile is one token's 128 heads.
    w, inp = _case(2, 128, 1, [5, 3], [60, 0], seed=40)
    out, flags = _run(inp, w)
    assert flags == 0
    assert_parity(out.cpu(), _oracle(inp, w), "prefill R=128")


def test_parity_paged():
    w, inp = _case(3, 64, 8, [130, 64, 1], [70, 0, 200], page=W.PAGE_SIZE, seed=41)
    out, flags = _run(inp, w)
    assert flags == 0
    assert_parity(out.cpu(), _oracle(inp, w), "prefill paged")


def test_parity_bf16_output():
    w, inp = _case(2, 32, 8, [150, 40], [20, 500], seed=42)
    out, flags = _run(inp, w, out_dtype=torch.bfloat16)
    assert flags == 0 and out.dtype == torch.bfloat16
    assert_parity(out.cpu(), _oracle(inp, w), "prefill bf16 out")


def test_parity_long_fresh_prompt():
    # 1000 tokens, R = 4: 32 query tiles per KV head, up to 8 key steps each.
    w, inp = _case(1, 8, 2, [1000], [0], seed=43)
    out, flags = _run(inp, w)
    assert flags == 0
    assert_parity(out.cpu(), _oracle(inp, w), "prefill 1000 fresh")


def test_generous_max_q_len_changes_nothing():
    w, inp = _case(2, 16, 2, [33, 7], [5, 100], seed=44)
    a, fa = _run(inp, w)
    b, fb = _run(inp, w, max_q=500)
    assert fa == fb == 0
    assert torch.equal(a, b)


def test_invalid_span_is_flagged_and_skipped():
    # Sequence 1 claims 9 new tokens but holds only 4: skipped, flagged; the
    # others are still computed.
    w, inp = _case(3, 16, 4, [6, 4, 5], [10, 0, 3], seed=45)
    cu = inp["cu_q"].clone()
    bad = dict(inp)
    bad["seq_lens"] = inp["seq_lens"].clone()
    bad["seq_lens"][1] = 3
    out, flags = _run(bad, w, cu=cu)
    assert flags & FLAG_BAD_QUERY_SPAN
    ref = _oracle(inp, w)
    good = np.r_[0:6, 10:15]
    assert_parity(out.cpu()[good], ref[good], "rows of valid sequences")


@pytest.mark.parametrize("name", sorted(W.PREFILL_WORKLOADS))
def test_full_size_sampled(name):
    # The benchmark's workloads at full size, in the launch it times; sampled
    # rows include every sequence's first and last tokens and tile edges.
    w = W.PREFILL_WORKLOADS[name]
    inp = W.make_prefill_inputs(w, pad_value=float("nan"))
    out, flags = _run(inp, w, out_dtype=torch.bfloat16)
    assert flags == 0
    cu = inp["cu_q"].numpy()
    rng = np.random.default_rng(7)
    rows = []
    for b in range(w.B):
        lo, hi = int(cu[b]), int(cu[b + 1])
        TQ = 128 // w.R
        picks = {lo, hi - 1, min(hi - 1, lo + TQ - 1), min(hi - 1, lo + TQ)} | set(rng.integers(lo, hi, 6).tolist())
        for i in sorted(picks):
            for h in {0, w.H_Q - 1, int(rng.integers(0, w.H_Q))}:
                rows.append((i, h))
    ref = _oracle(inp, w, rows=rows)
    got = torch.stack([out[i, h] for i, h in rows]).cpu()
    assert_parity(got, ref, name)
