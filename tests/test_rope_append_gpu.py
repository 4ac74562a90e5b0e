"""GPU parity of gqa_rope_append (rotary embedding + KV append) against the oracle.

RoPE follows "Grouped-Query Attention (GQA) and Multi-Query Attention (MQA):
Mathematical Foundations, ...", section 4 (RoPE on every query head and once
on every key head).  The kernel evaluates angles and rotations in double and
rounds once to the storage type; the oracle rotates in double, so each stored
element must equal the oracle value rounded to the storage type, up to one
ulp where the two sides' last bits of sin/cos straddle a rounding boundary.
"""

import dataclasses

import numpy as np
import pytest
import torch

import gqa_mqa_kv_b200 as gq
import oracle
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs, to_pages
from tests.helpers import assert_parity, to_device

pytestmark = pytest.mark.gpu


def new_token(B, H_Q, H_KV, D, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    mk = lambda *s: torch.randn(*s, generator=g).to(dtype)  # noqa: E731
    return mk(B, H_Q, D), mk(B, H_KV, D), mk(B, H_KV, D)


def assert_within_one_ulp(got: torch.Tensor, ref64: np.ndarray):
    ref = torch.from_numpy(ref64).to(got.dtype)  # RNE rounding of the oracle value
    g = got.cpu().float().double().numpy()
    r = ref.float().double().numpy()
    ulp = np.spacing(np.abs(r).astype(np.float32)).astype(np.float64)
    if got.dtype == torch.bfloat16:
        ulp *= 65536.0
    bad = np.abs(g - r) > ulp
    assert not bad.any(), f"{int(bad.sum())} elements differ by more than one ulp"
    assert (g == r).mean() > 0.99


@pytest.mark.parametrize("pairing", ["adjacent", "halves"])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_rope_and_append_contiguous(cuda_device, pairing, dtype):
    B, H_Q, H_KV, D, S = 4, 16, 4, 128, 300
    k_cache = torch.randn(B, S, H_KV, D).to(dtype)
    v_cache = torch.randn(B, S, H_KV, D).to(dtype)
    q, kn, vn = new_token(B, H_Q, H_KV, D, dtype, 1)
    pos = torch.tensor([0, 1, 177, 299], dtype=torch.int32)
    d = dict(q=q, kn=kn, vn=vn, kc=k_cache.clone(), vc=v_cache.clone(), pos=pos)
    d = {k: v.to(cuda_device) for k, v in d.items()}
    lens_out = torch.zeros(B, dtype=torch.int32, device=cuda_device)
    q_out = gq.gqa_rope_append(d["q"], d["kn"], d["vn"], d["pos"], d["kc"], d["vc"], rope_base=500000.0,
                               pairing=pairing, seq_lens_out=lens_out)
    torch.cuda.synchronize(cuda_device)
    assert_within_one_ulp(q_out, oracle.rope(q, pos, base=500000.0, pairing=pairing))
    k_ref = oracle.rope(kn, pos, base=500000.0, pairing=pairing)
    kc, vc = d["kc"].cpu(), d["vc"].cpu()
    expect_k, expect_v = k_cache.clone(), v_cache.clone()
    for b in range(B):
        m = int(pos[b])
        assert_within_one_ulp(kc[b, m], k_ref[b])
        expect_k[b, m] = kc[b, m]
        expect_v[b, m] = vn[b]
    assert torch.equal(kc, expect_k)  # no other row touched
    assert torch.equal(vc, expect_v)
    assert lens_out.cpu().tolist() == [1, 2, 178, 300]


def test_rope_and_append_paged_in_place(cuda_device):
    B, H_Q, H_KV, D = 3, 64, 8, 128
    w = dataclasses.replace(WORKLOADS["paged_long"], B=B, seq_len=640)
    inp = make_inputs(w)
    table = inp["block_table"]
    q, kn, vn = new_token(B, H_Q, H_KV, D, torch.bfloat16, 2)
    pos = torch.tensor([0, 64, 639], dtype=torch.int32)
    dq = q.to(cuda_device)
    kp, vp = inp["k_paged"].to(cuda_device), inp["v_paged"].to(cuda_device)
    out = gq.gqa_rope_append(dq, kn.to(cuda_device), vn.to(cuda_device), pos.to(cuda_device), kp, vp,
                             table.to(cuda_device), q_out=dq)
    torch.cuda.synchronize(cuda_device)
    assert out.data_ptr() == dq.data_ptr()
    assert_within_one_ulp(dq, oracle.rope(q, pos))
    k_ref = oracle.rope(kn, pos)
    kp, vp = kp.cpu(), vp.cpu()
    for b in range(B):
        m = int(pos[b])
        page, slot = int(table[b, m // 64]), m % 64
        assert_within_one_ulp(kp[page, slot], k_ref[b])
        assert torch.equal(vp[page, slot], vn[b])


def test_append_then_decode_matches_oracle(cuda_device):
    """A full decode step: RoPE + append the new token, then attend over L_b + 1 tokens."""
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged"], B=4, seq_len=1000)
    lens = torch.tensor([0, 63, 500, 999], dtype=torch.int32)
    inp = make_inputs(w, seq_lens=lens)
    q, kn, vn = new_token(w.B, w.H_Q, w.H_KV, w.D, torch.bfloat16, 3)
    d = to_device(inp, cuda_device)
    new_lens = torch.zeros_like(d["seq_lens"])
    q_rot = gq.gqa_rope_append(q.to(cuda_device), kn.to(cuda_device), vn.to(cuda_device), d["seq_lens"],
                               d["k"], d["v"], seq_lens_out=new_lens)
    out = gq.gqa_decode(q_rot, d["k"], d["v"], new_lens, scale=w.softmax_scale)
    torch.cuda.synchronize(cuda_device)
    # oracle side: rotate in double, round to the cache's bf16 exactly as stored, then attend
    q_ref = torch.from_numpy(oracle.rope(q, lens)).to(torch.bfloat16)
    k_ref = torch.from_numpy(oracle.rope(kn, lens)).to(torch.bfloat16)
    k, v = inp["k"].clone(), inp["v"].clone()
    for b in range(w.B):
        k[b, int(lens[b])] = k_ref[b]
        v[b, int(lens[b])] = vn[b]
    ref = oracle.gqa_decode(q_ref, k, v, lens + 1, w.softmax_scale)
    assert new_lens.cpu().tolist() == (lens + 1).tolist()
    assert_parity(out.cpu(), ref, "append + decode")


def test_bad_position_skips_the_write_and_raises_a_flag(cuda_device):
    B, H_Q, H_KV, D, S = 2, 8, 2, 64, 100
    kc = torch.zeros(B, S, H_KV, D, dtype=torch.bfloat16, device=cuda_device)
    vc = torch.zeros_like(kc)
    q, kn, vn = new_token(B, H_Q, H_KV, D, torch.bfloat16, 4)
    pos = torch.tensor([100, 5], dtype=torch.int32, device=cuda_device)  # 100 == capacity
    params = gq.make_params(q.to(cuda_device), kc, pos)
    ws = torch.zeros(gq.workspace_bytes(params), dtype=torch.uint8, device=cuda_device)
    gq.gqa_rope_append(q.to(cuda_device), kn.to(cuda_device), vn.to(cuda_device), pos, kc, vc, workspace=ws)
    assert gq.read_status(ws) & gq.FLAG_BAD_POSITION
    assert torch.count_nonzero(kc[0]) == 0 and torch.count_nonzero(kc[1, 5]) > 0
