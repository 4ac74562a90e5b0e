"""GPU parity: the CUDA path through the C ABI against the fp64 CPU oracle.

Reduced sizes are compared element by element (several tiles, ragged
tails, every grouping from MHA to MQA); the full benchmark-size workloads are
compared on sampled (batch, head) outputs that the oracle computes one by one.
Both sides read the same seeded inputs (gqa_mqa_kv_b200.workloads).
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


def run_gpu(inp, w, dev, paged=False, out_dtype=torch.float32, seq_lens=None, kernel="auto"):
    d = to_device(inp, dev)
    lens = d["seq_lens"] if seq_lens is None else seq_lens.to(dev)
    k, v = (d["k_paged"], d["v_paged"]) if paged else (d["k"], d["v"])
    table = d["block_table"] if paged else None
    ws = gq.make_workspace(gq.make_params(d["q"], k, lens, table, out_dtype), dev)
    out = gq.gqa_decode(d["q"], k, v, lens, table, scale=w.softmax_scale, out_dtype=out_dtype, workspace=ws,
                        kernel=kernel)
    assert gq.read_status(ws) & gq.FLAG_TIMEOUT == 0, "a pipeline wait timed out"
    return out.cpu()


def oracle_full(inp, w):
    return oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale)


def small(name, **kw):
    return dataclasses.replace(WORKLOADS[name], **kw)


# ------------------------------------------------------------ element-by-element

def test_tiny_fp32(cuda_device):
    w = WORKLOADS["tiny"]
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device), oracle_full(inp, w), "tiny fp32")


def test_tiny_bf16_copy_on_tensor_cores(cuda_device):
    w = dataclasses.replace(WORKLOADS["tiny"], dtype="bf16")
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device), oracle_full(inp, w), "tiny bf16")


def test_llama3_8b_full_size(cuda_device):
    w = WORKLOADS["llama3_8b"]
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device), oracle_full(inp, w), "llama3_8b")


@pytest.mark.parametrize("h_kv", [32, 8, 4, 2, 1])
def test_grouping_sweep_reduced(cuda_device, h_kv):
    w = small(f"sweep_hkv{h_kv}", B=4, seq_len=1000)  # 15 full tiles + a 40-token tail
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device), oracle_full(inp, w), f"sweep H_KV={h_kv}")


def test_ragged_with_edge_lengths(cuda_device):
    w = small("llama2_70b_ragged", B=12, seq_len=3000)
    lens = torch.tensor([0, 1, 63, 64, 65, 127, 128, 129, 3000, 2999, 1777, 5], dtype=torch.int32)
    inp = make_inputs(w, pad_value=float("nan"), seq_lens=lens)
    out = run_gpu(inp, w, cuda_device)
    assert torch.all(out[0] == 0)
    assert_parity(out, oracle_full(inp, w), "ragged edges")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_paged_reduced_and_bitwise_equal_to_contiguous(cuda_device, out_dtype):
    w = small("paged_long", B=3, seq_len=2000)  # 32 pages per sequence, last one partial
    inp = make_inputs(w, pad_value=float("nan"))
    paged = run_gpu(inp, w, cuda_device, paged=True, out_dtype=out_dtype)
    contig = run_gpu(inp, w, cuda_device, paged=False, out_dtype=out_dtype)
    assert torch.equal(paged.view(torch.int32 if out_dtype == torch.float32 else torch.int16),
                       contig.view(torch.int32 if out_dtype == torch.float32 else torch.int16))
    assert_parity(paged, oracle_full(inp, w), "paged")


def test_paged_ragged_lengths(cuda_device):
    w = small("paged_long", B=5, seq_len=1024)
    lens = torch.tensor([1024, 1, 64, 65, 700], dtype=torch.int32)
    inp = make_inputs(w, pad_value=float("nan"), seq_lens=lens)
    assert_parity(run_gpu(inp, w, cuda_device, paged=True), oracle_full(inp, w), "paged ragged")


@pytest.mark.parametrize("h_q,h_kv,d", [(8, 1, 64), (32, 1, 64), (16, 16, 64), (48, 1, 128),
                                        (40, 2, 128), (12, 3, 128), (6, 6, 128)])
def test_other_group_shapes(cuda_device, h_q, h_kv, d):
    w = dataclasses.replace(WORKLOADS["llama3_8b"], name="shape", B=3, H_Q=h_q, H_KV=h_kv, D=d,
                            seq_len=777, ragged=True)
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device), oracle_full(inp, w), f"{h_q}/{h_kv}/{d}")


def test_wide_group_beyond_tensor_core_path(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama3_8b"], name="wide", B=2, H_Q=128, H_KV=1, seq_len=300)
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device), oracle_full(inp, w), "R=128")


def test_fp32_paged(cuda_device):
    w = dataclasses.replace(WORKLOADS["tiny"], name="tinypaged", B=2, seq_len=320, page_size=64)
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device, paged=True), oracle_full(inp, w), "fp32 paged")


@pytest.mark.parametrize("name", ["llama3_8b", "sweep_hkv1"])
def test_bf16_output(cuda_device, name):
    w = small(name, B=2, seq_len=1500)
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device, out_dtype=torch.bfloat16), oracle_full(inp, w),
                  f"{name} bf16 out")


# ------------------------------------------------------------ closed forms on the GPU

def test_length_one_returns_v_exactly(cuda_device):
    w = small("llama3_8b", B=3, seq_len=64)
    inp = make_inputs(w, seq_lens=torch.ones(3, dtype=torch.int32))
    out = run_gpu(inp, w, cuda_device)
    R = w.R
    for h in range(w.H_Q):
        assert torch.equal(out[:, h, :], inp["v"][:, 0, h // R, :].float())


def test_one_hot_spike_selects_exactly(cuda_device):
    w = small("llama2_70b_ragged", B=2, seq_len=600)
    inp = make_inputs(w, seq_lens=torch.tensor([600, 333], dtype=torch.int32))
    inp["q"].fill_(1.0)
    inp["k"].zero_()
    spikes = {}
    rng = np.random.default_rng(5)
    for b in range(2):
        for g in range(w.H_KV):
            t = int(rng.integers(0, int(inp["seq_lens"][b])))
            spikes[(b, g)] = t
            inp["k"][b, t, g, :] = 20.0  # score gap ~226 in natural units
    out = run_gpu(inp, w, cuda_device)
    for (b, g), t in spikes.items():
        for r in range(w.R):
            assert torch.equal(out[b, g * w.R + r], inp["v"][b, t, g].float())


def test_group_map_probe(cuda_device):
    w = small("sweep_hkv4", B=2, seq_len=200)
    inp = make_inputs(w)
    for g in range(w.H_KV):
        inp["v"][:, :, g, :] = float(g)
    out = run_gpu(inp, w, cuda_device)
    for h in range(w.H_Q):
        assert torch.allclose(out[:, h, :], torch.full_like(out[:, h, :], h // w.R), atol=1e-4, rtol=0)


def test_paged_index_probe_bit_exact(cuda_device):
    """V encodes the logical token position; a key spike picks one token per
    (sequence, KV head); the output must decode to exactly that position."""
    w = small("paged_long", B=2, seq_len=8192)
    inp = make_inputs(w)
    T = inp["k"].shape[1]
    t = torch.arange(T)
    code = torch.stack([t % 64, (t // 64) % 64, t // 4096], dim=1).to(torch.bfloat16)
    v = torch.zeros_like(inp["v"])
    v[:, :, :, 0:3] = code[None, :, None, :]
    k = torch.zeros_like(inp["k"])
    q = torch.ones_like(inp["q"])
    targets = {(0, 0): 0, (0, 1): 63, (0, 2): 64, (0, 3): 8191, (0, 4): 4096, (0, 5): 4095,
               (0, 6): 127, (0, 7): 5000, (1, 0): 8191, (1, 1): 1, (1, 2): 2048, (1, 3): 6143,
               (1, 4): 6144, (1, 5): 65, (1, 6): 7000, (1, 7): 333}
    for (b, g), tt in targets.items():
        k[b, tt, g, :] = 20.0
    inp.update(q=q, k=k, v=v, k_paged=to_pages(k, inp["block_table"], 64),
               v_paged=to_pages(v, inp["block_table"], 64))
    out = run_gpu(inp, w, cuda_device, paged=True)
    for (b, g), tt in targets.items():
        for r in range(w.R):
            got = out[b, g * w.R + r, 0:3]
            assert got.tolist() == [tt % 64, (tt // 64) % 64, tt // 4096], (b, g, tt, got)


# ------------------------------------------------------------ device status flags

def test_clean_run_raises_no_flag(cuda_device):
    w = small("llama3_8b", B=2, seq_len=256)
    d = to_device(make_inputs(w), cuda_device)
    params = gq.make_params(d["q"], d["k"], d["seq_lens"])
    ws = torch.zeros(gq.workspace_bytes(params), dtype=torch.uint8, device=cuda_device)
    gq.gqa_decode(d["q"], d["k"], d["v"], d["seq_lens"], workspace=ws)
    assert gq.read_status(ws) == 0


def test_seq_len_clamped_and_flagged(cuda_device):
    w = small("llama3_8b", B=2, seq_len=256)
    inp = make_inputs(w)
    d = to_device(inp, cuda_device)
    params = gq.make_params(d["q"], d["k"], d["seq_lens"])
    ws = torch.zeros(gq.workspace_bytes(params), dtype=torch.uint8, device=cuda_device)
    bad = torch.tensor([300, -4], dtype=torch.int32, device=cuda_device)
    out = gq.gqa_decode(d["q"], d["k"], d["v"], bad, workspace=ws)
    assert gq.read_status(ws, clear=True) & gq.FLAG_SEQ_LEN_CLAMPED
    assert gq.read_status(ws) == 0
    ref = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], torch.tensor([256, 0], dtype=torch.int32),
                            w.softmax_scale)
    assert_parity(out.cpu(), ref, "clamped")


def test_bad_block_flagged_and_read_as_zeros(cuda_device):
    w = small("paged_long", B=2, seq_len=256)
    inp = make_inputs(w)
    d = to_device(inp, cuda_device)
    table = d["block_table"].clone()
    table[0, 1] = w.num_blocks + 7  # beyond the cache
    table[1, 2] = -1
    params = gq.make_params(d["q"], d["k_paged"], d["seq_lens"], table)
    ws = torch.zeros(gq.workspace_bytes(params), dtype=torch.uint8, device=cuda_device)
    out = gq.gqa_decode(d["q"], d["k_paged"], d["v_paged"], d["seq_lens"], table, workspace=ws)
    assert gq.read_status(ws) & gq.FLAG_BAD_BLOCK
    k, v = inp["k"].clone(), inp["v"].clone()
    k[0, 64:128] = 0
    v[0, 64:128] = 0
    k[1, 128:192] = 0
    v[1, 128:192] = 0
    ref = oracle.gqa_decode(inp["q"], k, v, inp["seq_lens"], w.softmax_scale)
    assert_parity(out.cpu(), ref, "bad block")


def test_repeated_calls_are_bitwise_identical(cuda_device):
    w = small("llama2_70b_ragged", B=6, seq_len=5000)
    d = to_device(make_inputs(w), cuda_device)
    a = gq.gqa_decode(d["q"], d["k"], d["v"], d["seq_lens"]).clone()
    b = gq.gqa_decode(d["q"], d["k"], d["v"], d["seq_lens"])
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


@pytest.mark.parametrize("kernel,h_q", [("mma_sync", 8), ("tcgen05", 32), ("auto", 128)])
def test_one_sequence_cut_across_every_cta(cuda_device, kernel, h_q):
    # One unit spread over all CTAs: every CTA holds a partial of it and the last
    # writer merges up to a grid's worth of partials inside the split kernel.
    w = small("llama2_70b_ragged", B=1, H_Q=h_q, H_KV=1, seq_len=148 * 64 * 3 + 17, ragged=False)
    inp = make_inputs(w)
    assert_parity(run_gpu(inp, w, cuda_device, kernel=kernel), oracle_full(inp, w), f"one sequence, {kernel}")


def test_merge_counters_over_many_calls_on_one_workspace(cuda_device):
    # Successive calls alternate between the two banks of merge counters; each
    # call's batch is cut differently, and every result must match the oracle.
    base = small("llama2_70b_ragged", B=5, seq_len=3000)
    ws = None
    for i in range(5):
        w = dataclasses.replace(base, seed=700 + i)
        inp = make_inputs(w)
        inp["seq_lens"][i % w.B] = 0  # an empty sequence somewhere in every call
        d = to_device(inp, cuda_device)
        if ws is None:
            ws = torch.zeros(gq.workspace_bytes(gq.make_params(d["q"], d["k"], d["seq_lens"])), dtype=torch.uint8,
                             device=cuda_device)
        out = torch.full(d["q"].shape, float("nan"), device=cuda_device)
        gq.gqa_decode(d["q"], d["k"], d["v"], d["seq_lens"], scale=w.softmax_scale, out=out, workspace=ws)
        assert_parity(out.cpu(), oracle_full(inp, w), f"call {i}")
    assert gq.read_status(ws) == 0


# ------------------------------------------------------------ full benchmark sizes, sampled

def sampled_pairs(w, lens, per_seq=4, seed=0):
    rng = np.random.default_rng(seed)
    pairs = []
    for b in range(w.B):
        heads = {0, w.H_Q - 1}
        while len(heads) < per_seq:
            heads.add(int(rng.integers(0, w.H_Q)))
        pairs += [(b, h) for h in sorted(heads)]
    return pairs


def check_sampled(out, inp, w, pairs):
    ref = oracle.gqa_decode(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale, pairs=pairs)
    got = torch.stack([out[b, h] for b, h in pairs])
    assert_parity(got, ref, f"{w.name} sampled")


@pytest.mark.parametrize("name", ["llama2_70b_ragged", "paged_long", "sweep_hkv32", "sweep_hkv8", "sweep_hkv4",
                                  "sweep_hkv2", "sweep_hkv1"])
def test_full_size_sampled(cuda_device, name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    out = run_gpu(inp, w, cuda_device, paged=bool(w.page_size))
    assert torch.all(torch.isfinite(out))
    check_sampled(out, inp, w, sampled_pairs(w, inp["seq_lens"], per_seq=4 if w.B > 8 else 8))
