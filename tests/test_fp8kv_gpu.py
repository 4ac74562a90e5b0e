"""GPU parity of gqa_decode_fp8kv (E4M3 cache, per-KV-head scales) against the oracle.

The oracle decodes the same E4M3 bytes exactly and multiplies by the same
scales, so the comparison isolates the kernel's arithmetic from quantisation:
the tolerance is the one every other parity test uses.
"""

import dataclasses

import numpy as np
import pytest
import torch

import gqa_mqa_kv_b200 as gq
import oracle
from gqa_mqa_kv_b200.workloads import WORKLOADS, make_inputs
from tests.helpers import assert_parity, to_device

pytestmark = pytest.mark.gpu


def run_fp8(inp, w, dev, paged=False, out_dtype=torch.float32, kernel="auto"):
    d = to_device(inp, dev)
    k = d["k_paged"] if paged else d["k"]
    v = d["v_paged"] if paged else d["v"]
    table = d["block_table"] if paged else None
    params = gq.make_params(d["q"], k, d["seq_lens"], table, out_dtype)
    ws = gq.make_workspace(params, dev)
    out = gq.gqa_decode_fp8kv(d["q"], k, v, d["k_scale"], d["v_scale"], d["seq_lens"], table,
                              scale=w.softmax_scale, out_dtype=out_dtype, workspace=ws, kernel=kernel)
    assert gq.read_status(ws) & gq.FLAG_TIMEOUT == 0, "a pipeline wait timed out"
    return out.cpu()


def ref_fp8(inp, w, pairs=None):
    return oracle.gqa_decode_scaled(inp["q"], inp["k"], inp["v"], inp["seq_lens"], w.softmax_scale,
                                    inp["k_scale"], inp["v_scale"], pairs=pairs)


def test_fp8_contiguous_ragged_with_edges(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged_fp8"], B=8, seq_len=3000)
    lens = torch.tensor([0, 1, 63, 64, 65, 1777, 3000, 129], dtype=torch.int32)
    inp = make_inputs(w, pad_value=float("nan"), seq_lens=lens)
    out = run_fp8(inp, w, cuda_device)
    assert torch.all(out[0] == 0)
    assert_parity(out, ref_fp8(inp, w), "fp8 contiguous")


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16])
def test_fp8_paged_equals_contiguous_bitwise(cuda_device, out_dtype):
    w = dataclasses.replace(WORKLOADS["paged_long_fp8"], B=3, seq_len=2000)
    inp = make_inputs(w, pad_value=float("nan"))
    paged = run_fp8(inp, w, cuda_device, paged=True, out_dtype=out_dtype)
    contig = run_fp8(inp, w, cuda_device, paged=False, out_dtype=out_dtype)
    iv = torch.int32 if out_dtype == torch.float32 else torch.int16
    assert torch.equal(paged.view(iv), contig.view(iv))
    assert_parity(paged, ref_fp8(inp, w), "fp8 paged")


@pytest.mark.parametrize("h_q,h_kv,d", [(32, 8, 128), (64, 4, 128), (64, 2, 128), (32, 1, 128), (24, 1, 128),
                                        (16, 4, 64), (8, 1, 64), (64, 1, 128)])
def test_fp8_group_shapes(cuda_device, h_q, h_kv, d):
    """R <= 32 at head_dim 128 runs on the tcgen05 kernel; the rest on CUDA cores."""
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged_fp8"], name="shape", B=3, H_Q=h_q, H_KV=h_kv,
                            D=d, seq_len=700)
    inp = make_inputs(w)
    assert_parity(run_fp8(inp, w, cuda_device), ref_fp8(inp, w), f"fp8 {h_q}/{h_kv}/{d}")


def test_fp8_one_hot_spike_returns_the_scaled_value(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged_fp8"], B=2, seq_len=300)
    inp = make_inputs(w, seq_lens=torch.tensor([300, 77], dtype=torch.int32))
    inp["q"].fill_(1.0)
    k8 = torch.zeros(inp["k"].shape, dtype=torch.uint8)
    spikes = {(0, 3): 299, (1, 5): 0, (1, 0): 76}
    for (b, g), t in spikes.items():
        k8[b, t, g, :] = 0x7E  # 448
    inp["k"] = k8.view(torch.float8_e4m3fn)
    out = run_fp8(inp, w, cuda_device)
    for (b, g), t in spikes.items():
        expect = inp["v"][b, t, g].float() * inp["v_scale"][g]
        assert torch.allclose(out[b, g * w.R], expect, rtol=1e-6, atol=0)


def test_fp8_full_size_sampled(cuda_device):
    w = WORKLOADS["llama2_70b_ragged_fp8"]
    inp = make_inputs(w)
    out = run_fp8(inp, w, cuda_device)
    rng = np.random.default_rng(0)
    pairs = [(b, int(h)) for b in range(w.B) for h in {0, w.H_Q - 1, int(rng.integers(0, w.H_Q))}]
    got = torch.stack([out[b, h] for b, h in pairs])
    assert_parity(got, ref_fp8(inp, w, pairs=pairs), "fp8 full size")


@pytest.mark.parametrize("kernel,h_q", [("tcgen05", 8), ("tcgen05", 32), ("mma_sync", 8)])
def test_fp8_one_sequence_cut_across_every_cta(cuda_device, kernel, h_q):
    # One unit spread over all CTAs, with a ragged tail: every CTA holds a
    # partial and the last writer merges a grid's worth of them.
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged_fp8"], name="one", B=1, H_Q=h_q, H_KV=1,
                            seq_len=148 * 64 * 3 + 17, ragged=False)
    inp = make_inputs(w)
    assert_parity(run_fp8(inp, w, cuda_device, kernel=kernel), ref_fp8(inp, w), f"fp8 one sequence, {kernel}")


@pytest.mark.parametrize("name", ["paged_long_fp8", "llama3_8b_fp8"])
def test_fp8_other_full_size_workloads_sampled(cuda_device, name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    out = run_fp8(inp, w, cuda_device, paged=bool(w.page_size))
    assert torch.all(torch.isfinite(out))
    rng = np.random.default_rng(1)
    pairs = [(b, int(h)) for b in range(w.B) for h in {0, w.H_Q - 1, int(rng.integers(0, w.H_Q))}]
    got = torch.stack([out[b, h] for b, h in pairs])
    assert_parity(got, ref_fp8(inp, w, pairs=pairs), f"{name} sampled")


def test_fp8_requires_bf16_query(cuda_device):
    w = dataclasses.replace(WORKLOADS["llama2_70b_ragged_fp8"], B=1, seq_len=64)
    d = to_device(make_inputs(w), cuda_device)
    with pytest.raises(ValueError):
        gq.gqa_decode_fp8kv(d["q"].float(), d["k"], d["v"], d["k_scale"], d["v_scale"], d["seq_lens"])
